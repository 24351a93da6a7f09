"""Multi-rank host logic on CPU (gloo, world size 2): batch sharding and the
summation of the shared-parameter gradients across ranks.

Each rank stands in for one GPU: it takes its own batch (or its shard of one
batch), computes per-rank gradients (here with the float64 oracle, since there is
no GPU), and the ranks all-reduce dA and dD.  The result must equal the
gradients of the whole batch computed in one process.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from semi_markov_crf_prefix_b200.dist import reduce_param_grads, shard_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_batch(rank):
    """Rank `rank`'s batch: its own emissions and lengths, parameters of seed 0."""
    import semicrf_workloads as wl
    base = wl.make_workload("ner", seed=0, B=4, T=64)
    own = wl.make_workload("ner", seed=100 + rank, B=4, T=64)
    base.x, base.lengths = own.x, own.lengths
    return base


def _worker(rank, world, port, mode, out_dir):
    import oracle
    import semicrf_workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        if mode == "weak":        # every rank its own data, parameters shared
            w = _rank_batch(rank)
            x, lengths = w.x, w.lengths
        else:                     # one batch split by sequence
            w = wl.make_workload("ner", seed=0, B=5, T=64)
            lo, hi = shard_range(w.B, world, rank)
            x, lengths = w.x[lo:hi], w.lengths[lo:hi]
        r = oracle.factorised(x, w.A, w.D, lengths, nthreads=1)
        dA = torch.from_numpy(r["dA"].copy())
        dD = torch.from_numpy(r["dD"].copy())
        reduce_param_grads(dA, dD)
        np.save(os.path.join(out_dir, f"dA_{rank}.npy"), dA.numpy())
        np.save(os.path.join(out_dir, f"dD_{rank}.npy"), dD.numpy())
        np.save(os.path.join(out_dir, f"logZ_{rank}.npy"), r["logZ"])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["weak", "shard"])
def test_two_rank_gradient_sum(tmp_path, mode):
    import oracle
    import semicrf_workloads as wl
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), mode, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    if mode == "weak":
        ws = [_rank_batch(r) for r in range(world)]
        x = np.concatenate([w.x for w in ws])
        lengths = np.concatenate([w.lengths for w in ws])
        ref = oracle.factorised(x, ws[0].A, ws[0].D, lengths)
    else:
        w = wl.make_workload("ner", seed=0, B=5, T=64)
        ref = oracle.factorised(w.x, w.A, w.D, w.lengths)
    ref_dA, ref_dD = ref["dA"], ref["dD"]
    logZ = np.concatenate([np.load(tmp_path / f"logZ_{r}.npy") for r in range(world)])
    np.testing.assert_allclose(logZ, ref["logZ"], rtol=1e-13)
    for r in range(world):
        np.testing.assert_allclose(np.load(tmp_path / f"dA_{r}.npy"), ref_dA, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(np.load(tmp_path / f"dD_{r}.npy"), ref_dD, rtol=1e-12, atol=1e-12)


def test_shard_range_partitions():
    for B in (1, 2, 5, 32, 33):
        for world in (1, 2, 3, 8):
            spans = [shard_range(B, world, r) for r in range(world)]
            covered = [i for lo, hi in spans for i in range(lo, hi)]
            assert covered == list(range(B))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)
