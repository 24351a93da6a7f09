"""Full-size parity: the named long workloads at their full sizes, in the launch
configuration the benchmark times, against the float64 oracle.

* large-label (B=4, T=200 000, K=512, C=256) and genomic (B=1, T=100 000,
  K=1000, C=24): log Z, dA, dD and the Viterbi result element by element, dX
  at every position (genomic) or at every 128th position plus the first and
  last 256 of each sequence (large-label), for both ways of computing the
  gradients: the fused step (semicrf_forward_backward) and the checkpointed
  pair (semicrf_forward + semicrf_backward);
* the million-position scale recipe (K=200, C=24) at T=50 000: the same
  comparison.

The oracle's results come from ``tests/oracle_cache.py`` (a script that calls
only the oracle), because the large-label workload takes the float64 oracle
hours of CPU.  Without a stored result the genomic and scale comparisons run
the oracle here (minutes on 16 cores); the large-label one is skipped and says
how to write it.

Bars: relative 1e-5 on log Z, absolute 1e-4 on every gradient entry (the
counts dA, dD reach 10^3-10^5 here; the scaled error |d|/max(1,|g|) is
reported beside the absolute one), Viterbi score and labels exact, segment
starts exact or a valid optimal segmentation (an exact tie, see
check_viterbi in test_gpu_parity.py).
"""
import numpy as np
import pytest

import oracle
import oracle_cache
from test_gpu_parity import GRAD_ATOL, LOGZ_RTOL, check_viterbi

pytestmark = pytest.mark.gpu


def _oracle_result(name):
    r = oracle_cache.load(name)
    if r is not None:
        return r
    if name == "large":
        pytest.skip("no stored oracle result for the large-label workload "
                    "(python tests/oracle_cache.py large writes it; about 2 h on 8 cores)")
    w = oracle_cache.workload(name)
    o = oracle.factorised(w.x, w.A, w.D, w.lengths)
    score, labels, seg = oracle.viterbi(w.x, w.A, w.D, w.lengths)
    return dict(logZ=o["logZ"], dA=o["dA"], dD=o["dD"], dX=o["dX"], dx_pos=np.arange(w.T),
                score=score, labels=labels, seg_start=seg)


def _gpu_both_paths(w):
    """prefix_scan, then the fused step and the checkpointed pair on one
    workspace, then Viterbi; numpy results of each."""
    import torch
    import semi_markov_crf_prefix_b200 as sc
    dev = torch.device("cuda:0")
    x = torch.from_numpy(w.x).to(dev)
    A = torch.from_numpy(w.A).to(dev)
    D = torch.from_numpy(w.D).to(dev)
    lens = torch.from_numpy(w.lengths).to(dev)
    ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
    sc.clear_device_status(ws)
    S, _ = sc.prefix_scan(x, lens, ws=ws)
    out = {}
    logZ, dX, dA, dD, _ = sc.forward_backward(S, A, D, lens, ws=ws)
    out["fused"] = dict(logZ=logZ.cpu().numpy(), dX=dX.cpu().numpy(), dA=dA.cpu().numpy(), dD=dD.cpu().numpy(),
                        status=sc.device_status(ws))
    del dX
    logZ, _ = sc.forward(S, A, D, lens, ws=ws)
    dX, dA, dD = sc.backward(S, A, D, lens, ws)
    out["ckpt"] = dict(logZ=logZ.cpu().numpy(), dX=dX.cpu().numpy(), dA=dA.cpu().numpy(), dD=dD.cpu().numpy(),
                       status=sc.device_status(ws))
    del dX, ws
    torch.cuda.empty_cache()
    wsv = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_VITERBI, device=dev)
    sc.clear_device_status(wsv)
    score, labels, seg = sc.viterbi(S, A, D, lens, ws=wsv)
    out["viterbi"] = dict(score=score.cpu().numpy(), labels=labels.cpu().numpy(), seg_start=seg.cpu().numpy(),
                          status=sc.device_status(wsv))
    del wsv, S
    torch.cuda.empty_cache()
    return out


def _compare(name, w, r, g):
    report = []
    for path in ("fused", "ckpt"):
        o = g[path]
        assert o["status"] == 0, (path, o["status"])
        rel = np.abs(o["logZ"] - r["logZ"]) / np.abs(r["logZ"])
        assert rel.max() <= LOGZ_RTOL, (path, "logZ", rel.max())
        assert rel.max() <= 1e-10, (path, "precision logZ", rel.max())
        line = [f"{name} {path}: logZ rel {rel.max():.2e}"]
        for k in ("dA", "dD"):
            d = np.abs(o[k] - r[k])
            scaled = (d / np.maximum(1.0, np.abs(r[k]))).max()
            line.append(f"{k} abs {d.max():.2e} scaled {scaled:.2e} (max |{k}| {np.abs(r[k]).max():.3g})")
            assert d.max() <= GRAD_ATOL, (path, k, d.max(), scaled)
        pos = r["dx_pos"]
        d = np.abs(o["dX"][:, pos, :] - r["dX"])
        line.append(f"dX abs {d.max():.2e} at {len(pos)} positions x {w.B} sequences")
        assert d.max() <= GRAD_ATOL, (path, "dX", d.max())
        # invariants over every position (the ones not sampled above included)
        L = w.lengths.astype(np.int64)
        for b in range(w.B):
            np.testing.assert_allclose(o["dX"][b, :L[b]].sum(axis=1), 0.0, atol=1e-4)   # coverage sums to one
        dvec = np.arange(1, w.K + 1)[:, None]
        np.testing.assert_allclose((dvec * o["dD"]).sum(), L.sum(), rtol=1e-9)          # total length
        np.testing.assert_allclose(o["dD"].sum() - o["dA"].sum(), w.B, atol=1e-5)       # segments - transitions
        report.append("; ".join(line))
    # the two paths agree with each other more tightly than with the oracle
    a, b = g["fused"], g["ckpt"]
    np.testing.assert_allclose(a["logZ"], b["logZ"], rtol=1e-12)
    for k in ("dA", "dD"):
        np.testing.assert_allclose(a[k], b[k], atol=1e-6, rtol=1e-10)
    np.testing.assert_allclose(a["dX"], b["dX"], atol=1e-6, rtol=0)
    v = g["viterbi"]
    assert v["status"] == 0
    check_viterbi(w, v, ref=(r["score"], r["labels"], r["seg_start"]))
    same = sum(np.array_equal(v["seg_start"][b], r["seg_start"][b]) for b in range(w.B))
    report.append(f"{name} viterbi: score and labels exact, segment starts identical in {same} of {w.B}")
    print("\n" + "\n".join(report))


@pytest.mark.parametrize("name", ["large", "genomic", "stress50k"])
def test_full_size_against_oracle(name):
    r = _oracle_result(name)
    w = oracle_cache.workload(name)
    g = _gpu_both_paths(w)
    _compare(name, w, r, g)
