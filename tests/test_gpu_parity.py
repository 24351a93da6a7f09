"""GPU parity: the CUDA path through the C ABI against the float64 CPU oracle.

Tolerances (the stated bar): relative error <= 1e-5 on log Z, absolute error
<= 1e-4 on every gradient entry, bit-exact Viterbi labels and segment starts.
The path computes in float64, so the tests also hold it to tighter internal
bounds (marked "precision") that would catch a silent drop to float32.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import bruteforce as bf
import semicrf_workloads as wl

pytestmark = pytest.mark.gpu

LOGZ_RTOL = 1e-5
GRAD_ATOL = 1e-4


def _torch():
    import torch
    return torch


def run_gpu(w, ckpt_interval=0, grad=None, x=None, lengths=None):
    """prefix_scan + forward + backward + viterbi on cuda:0; numpy results."""
    torch = _torch()
    import semi_markov_crf_prefix_b200 as sc
    dev = torch.device("cuda:0")
    xs = torch.from_numpy(np.ascontiguousarray(w.x if x is None else x)).to(dev)
    A = torch.from_numpy(w.A).to(dev)
    D = torch.from_numpy(w.D).to(dev)
    lens = torch.from_numpy(np.ascontiguousarray(w.lengths if lengths is None else lengths)).to(dev)
    g = None if grad is None else torch.from_numpy(np.asarray(grad, np.float64)).to(dev)
    ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, ckpt_interval, device=dev)
    sc.clear_device_status(ws)
    S, nu = sc.prefix_scan(xs, lens, ws=ws)
    logZ, _ = sc.forward(S, A, D, lens, ws=ws, ckpt_interval=ckpt_interval)
    dX, dA, dD = sc.backward(S, A, D, lens, ws, grad_logZ=g, ckpt_interval=ckpt_interval)
    status = sc.device_status(ws)
    wsv = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_VITERBI, device=dev)
    sc.clear_device_status(wsv)
    score, labels, seg = sc.viterbi(S, A, D, lens, ws=wsv)
    vstatus = sc.device_status(wsv)
    torch.cuda.synchronize()
    return dict(S=S.cpu().numpy(), nu=nu.cpu().numpy(), logZ=logZ.cpu().numpy(), dX=dX.cpu().numpy(),
                dA=dA.cpu().numpy(), dD=dD.cpu().numpy(), score=score.cpu().numpy(),
                labels=labels.cpu().numpy(), seg_start=seg.cpu().numpy(), status=status,
                vstatus=vstatus)


def run_gpu_fused(w, grad=None):
    """prefix_scan + forward_backward (both chains side by side) on cuda:0."""
    torch = _torch()
    import semi_markov_crf_prefix_b200 as sc
    dev = torch.device("cuda:0")
    xs = torch.from_numpy(np.ascontiguousarray(w.x)).to(dev)
    A = torch.from_numpy(w.A).to(dev)
    D = torch.from_numpy(w.D).to(dev)
    lens = torch.from_numpy(np.ascontiguousarray(w.lengths)).to(dev)
    g = None if grad is None else torch.from_numpy(np.asarray(grad, np.float64)).to(dev)
    ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
    sc.clear_device_status(ws)
    S, nu = sc.prefix_scan(xs, lens, ws=ws)
    logZ, dX, dA, dD, _ = sc.forward_backward(S, A, D, lens, ws=ws, grad_logZ=g)
    status = sc.device_status(ws)
    wsv = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_VITERBI, device=dev)
    sc.clear_device_status(wsv)
    score, labels, seg = sc.viterbi(S, A, D, lens, ws=wsv)
    vstatus = sc.device_status(wsv)
    torch.cuda.synchronize()
    return dict(S=S.cpu().numpy(), nu=nu.cpu().numpy(), logZ=logZ.cpu().numpy(), dX=dX.cpu().numpy(),
                dA=dA.cpu().numpy(), dD=dD.cpu().numpy(), score=score.cpu().numpy(),
                labels=labels.cpu().numpy(), seg_start=seg.cpu().numpy(), status=status,
                vstatus=vstatus)


def check_against_oracle(w, g, grad=None, precision=True):
    o = oracle.factorised(w.x, w.A, w.D, w.lengths, grad_logZ=grad)
    assert g["status"] == 0 and g["vstatus"] == 0
    rel = np.abs(g["logZ"] - o["logZ"]) / np.abs(o["logZ"])
    assert rel.max() <= LOGZ_RTOL, rel.max()
    for k in ("dX", "dA", "dD"):
        err = np.abs(g[k] - o[k]).max()
        assert err <= GRAD_ATOL, (k, err)
    if precision:
        assert rel.max() <= 1e-11, ("precision logZ", rel.max())
        assert np.abs(g["dA"] - o["dA"]).max() <= 1e-8 * max(1.0, np.abs(o["dA"]).max())
        assert np.abs(g["dD"] - o["dD"]).max() <= 1e-8 * max(1.0, np.abs(o["dD"]).max())
        assert np.abs(g["dX"] - o["dX"]).max() <= 1e-6
    check_viterbi(w, g)
    return o


def check_viterbi(w, g, ref=None):
    """Viterbi against the oracle.  The best score is unique, and so are the
    per-position labels on continuous inputs.  The segment starts are not: two
    adjacent segments of one label with durations d and d' score exactly the same
    in either order (the prefix-sum differences telescope and the same D and A
    terms appear), so wherever the best path holds such a pair there is an exact
    tie, and the last bits of S -- summed in a different order on the two sides --
    pick which side wins.  So: score and labels as the oracle's; segment starts
    equal to the oracle's or, for a sequence where they differ, a valid
    segmentation whose score, recomputed by the oracle from the definition, is
    the optimum to rounding.  ref: the oracle's (score, labels, seg_start) when
    already computed."""
    s, labels, seg = oracle.viterbi(w.x, w.A, w.D, w.lengths) if ref is None else ref
    np.testing.assert_allclose(g["score"], s, rtol=1e-12)
    assert np.array_equal(g["labels"], labels)
    differ = [b for b in range(w.B) if not np.array_equal(g["seg_start"][b], seg[b])]
    if not differ:
        return
    rescored = oracle.path_score(w.x, w.A, w.D, w.lengths, g["labels"], g["seg_start"])
    for b in differ:
        L = int(w.lengths[b])
        st = g["seg_start"][b].astype(bool)
        assert st[0] and not st[L:].any(), b
        starts = np.flatnonzero(st[:L])
        assert np.diff(np.append(starts, L)).max() <= w.K, b
        for a, e in zip(starts, np.append(starts[1:], L)):
            assert np.all(g["labels"][b, a:e] == g["labels"][b, a]), b   # one label per segment
        assert abs(rescored[b] - s[b]) <= 1e-12 * max(1.0, abs(s[b])), (b, rescored[b], s[b])


def test_prefix_scan_matches_oracle():
    w = wl.make_workload("ner")
    g = run_gpu(w)
    S, nu = oracle.prefix(w.x, w.lengths)
    np.testing.assert_allclose(g["nu"], nu, rtol=0, atol=1e-13)
    np.testing.assert_allclose(g["S"], S, rtol=0, atol=1e-11)
    for b in range(w.B):
        L = int(w.lengths[b])
        assert np.all(g["S"][b, L:] == g["S"][b, L])
        assert abs(g["S"][b, L]).max() < 1e-10


def test_tiny10_against_enumeration():
    w = wl.make_workload("tiny10")
    g = run_gpu(w)
    e = bf.enumerate_batch(w.x, w.A, w.D, w.lengths)
    np.testing.assert_allclose(g["logZ"], e["logZ"], rtol=1e-12)
    np.testing.assert_allclose(g["dA"], e["dA"], atol=1e-11)
    np.testing.assert_allclose(g["dD"], e["dD"], atol=1e-11)
    np.testing.assert_allclose(g["dX"], e["dX"], atol=1e-6)
    np.testing.assert_allclose(g["score"], e["score"], rtol=1e-12)
    assert np.array_equal(g["labels"], e["labels"]) and np.array_equal(g["seg_start"], e["seg_start"])


@pytest.mark.parametrize("name", ["tiny", "ner"])
def test_named_small(name):
    w = wl.make_workload(name)
    check_against_oracle(w, run_gpu(w))


@pytest.mark.parametrize("name", ["tiny", "ner"])
def test_named_small_cluster_kernels(name, monkeypatch):
    # the same workloads through the cluster kernels instead of the warp-per-sequence ones
    monkeypatch.setenv("SEMICRF_KERNEL_PATH", "general")
    w = wl.make_workload(name)
    check_against_oracle(w, run_gpu(w))


@pytest.mark.parametrize("plan", ["1,0,0", "2,4,0", "4,0,1", "4,2,2", "8,0,0", "0,0,4"])
def test_cluster_geometries(plan, monkeypatch):
    # the cluster kernels under other splits of the labels over CTAs (G), of the
    # transition terms over lanes (LPL) and of the window rows over lanes (LPW)
    monkeypatch.setenv("SEMICRF_KERNEL_PATH", "general")
    monkeypatch.setenv("SEMICRF_CL_PLAN", plan)
    w = wl.random_small(seed=21, B=3, T=150, K=40, C=24, ragged=True)
    check_against_oracle(w, run_gpu(w))
    w = wl.random_small(seed=22, B=2, T=90, K=1, C=40, ragged=True)   # K = 1: duration-1 terms only
    if plan in ("1,0,0", "2,4,0", "8,0,0"):
        check_against_oracle(w, run_gpu(w))


@pytest.mark.parametrize("plan", ["12,0,0", "14,0,0", "16,8,16"])
def test_cluster_sizes_beyond_powers_of_two(plan, monkeypatch):
    # clusters of 12 and 14 CTAs (the planner's fallback when the power-of-two
    # clusters of a launch cannot all be resident), odd label counts per CTA
    # included (their exchange blocks carry a zero pad), on a small random
    # problem; and the large-label geometry at full K and C on a short sequence
    monkeypatch.setenv("SEMICRF_KERNEL_PATH", "general")
    monkeypatch.setenv("SEMICRF_CL_PLAN", plan)
    if plan.endswith(",0,0"):
        # 5 labels per CTA with 12 CTAs at C = 56; 4 and 3 with 14 at C = 56 and 41
        for C in {"12,0,0": (56,), "14,0,0": (56, 41)}[plan]:
            w = wl.random_small(seed=23, B=3, T=120, K=30, C=C, ragged=True)
            check_against_oracle(w, run_gpu(w))
            check_against_oracle(w, run_gpu_fused(w))
    else:
        w = wl.make_workload("large", B=1, T=700)
        check_against_oracle(w, run_gpu_fused(w))
        check_against_oracle(w, run_gpu(w))


def test_kernel_families_agree():
    import os
    w = wl.make_workload("ner", B=8)
    a = run_gpu(w)
    os.environ["SEMICRF_KERNEL_PATH"] = "general"
    try:
        b = run_gpu(w)
    finally:
        del os.environ["SEMICRF_KERNEL_PATH"]
    np.testing.assert_allclose(a["logZ"], b["logZ"], rtol=1e-13)
    for k in ("dA", "dD"):
        np.testing.assert_allclose(a[k], b[k], atol=1e-9, rtol=1e-12)
    # dX is float32: a float64 difference of ~1e-15 may flip one float32 rounding
    np.testing.assert_allclose(a["dX"], b["dX"], atol=2e-7, rtol=0)


def test_upstream_weights():
    w = wl.make_workload("ner")
    grad = np.random.default_rng(1).normal(size=w.B)
    check_against_oracle(w, run_gpu(w, grad=grad), grad=grad)


def test_speech_full():
    w = wl.make_workload("speech")
    check_against_oracle(w, run_gpu(w))


def test_genomic_reduced_T():
    w = wl.make_workload("genomic", T=6000)
    check_against_oracle(w, run_gpu(w))


def test_large_reduced_T():
    # full K and C (and so the full cluster layout) on a shorter sequence
    w = wl.make_workload("large", B=2, T=1500)
    check_against_oracle(w, run_gpu(w))


@pytest.mark.parametrize("seed,B,T,K,C", [(8, 9, 90, 32, 32), (9, 6, 130, 24, 9), (10, 5, 64, 31, 1),
                                           (11, 7, 200, 2, 31), (12, 3, 40, 17, 24),
                                           (0, 3, 37, 5, 3), (1, 5, 100, 1, 7), (2, 2, 70, 70, 2),
                                           (3, 4, 129, 33, 33), (4, 1, 1, 4, 5), (5, 2, 50, 200, 9),
                                           (6, 3, 300, 40, 64), (7, 2, 200, 300, 20)])
def test_random_shapes(seed, B, T, K, C):
    w = wl.random_small(seed, B, T, K, C, ragged=True)
    check_against_oracle(w, run_gpu(w))


def test_checkpoint_interval_invariance():
    w = wl.make_workload("ner", B=6)
    T, K = w.T, w.K
    ref = run_gpu(w, ckpt_interval=0)
    for ck in (1, 7, int(math.ceil(math.sqrt(T * K))), T):
        g = run_gpu(w, ckpt_interval=ck)
        for k in ("logZ", "dX", "dA", "dD"):
            assert np.array_equal(g[k], ref[k]), (ck, k)


def test_nan_padding_is_never_read():
    w = wl.make_workload("ner")
    ref = run_gpu(w)
    x = w.x.copy()
    for b in range(w.B):
        x[b, int(w.lengths[b]):] = np.nan
    g = run_gpu(w, x=x)
    for k in ("logZ", "dX", "dA", "dD", "score", "labels", "seg_start"):
        assert np.array_equal(g[k], ref[k]), k


def test_invalid_length_sets_device_status():
    w = wl.make_workload("tiny")
    bad = w.lengths.copy()
    bad[1] = w.T + 1
    g = run_gpu(w, lengths=bad)
    assert g["status"] == 7 and g["vstatus"] == 7


def test_zero_scores_closed_form_and_tie_break():
    L, K, C = 40, 6, 5
    w = wl.random_small(0, 1, L, K, C, ragged=False)
    w.x[:] = 0
    w.A[:] = 0
    w.D[:] = 0
    g = run_gpu(w)
    N = [1] + [0] * L
    for t in range(1, L + 1):
        N[t] = C * sum(N[t - d] for d in range(1, min(K, t) + 1))
    np.testing.assert_allclose(g["logZ"][0], math.log(N[L]), rtol=1e-13)
    assert g["score"][0] == 0.0
    assert np.all(g["labels"][0] == 0) and np.all(g["seg_start"][0] == 1)


def test_zero_scores_golden_at_workload_shapes():
    # all-zero scores at the named workloads' K and C, lengths up to 5000 (both
    # kernel families): log Z against the exact segmentation counts stored in
    # tests/golden/zero_scores.txt; every Viterbi candidate ties at score 0
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "zero_scores.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert len(rows) >= 4
    for L, K, C, z in rows:
        L, K, C, z = int(L), int(K), int(C), float(z)
        w = wl.random_small(0, 1, L, K, C, ragged=False)
        w.x[:] = 0
        w.A[:] = 0
        w.D[:] = 0
        g = run_gpu_fused(w)
        assert g["status"] == 0 and g["vstatus"] == 0, (L, K, C)
        np.testing.assert_allclose(g["logZ"][0], z, rtol=1e-12, err_msg=str((L, K, C)))
        assert g["score"][0] == 0.0


def test_genomic_full_size_invariants():
    """Full genomic size: log Z against the oracle forward, plus invariants of the
    gradients that hold at any size."""
    w = wl.make_workload("genomic")
    g = run_gpu(w)
    assert g["status"] == 0
    lz = oracle.logz(w.x, w.A, w.D, w.lengths)
    assert abs(g["logZ"][0] - lz[0]) / abs(lz[0]) <= 1e-11
    L = int(w.lengths[0])
    dvec = np.arange(1, w.K + 1)[:, None]
    np.testing.assert_allclose((dvec * g["dD"]).sum(), L, rtol=1e-10)         # total length
    np.testing.assert_allclose(g["dD"].sum() - g["dA"].sum(), 1.0, atol=1e-6)  # segments - transitions
    np.testing.assert_allclose(g["dX"][0, :L].sum(axis=1), 0.0, atol=1e-4)    # coverage sums to one
    np.testing.assert_allclose(g["dX"][0].sum(axis=0), 0.0, atol=1e-2)        # zero mean per label
    assert g["dA"].min() >= 0 and g["dD"].min() >= 0


def test_stress_million_positions():
    """Scale test, one sequence of 10^6 positions with K = 200, C = 24: gradient
    invariants at full size (they tie the forward and backward chains together at
    every position) and the Viterbi path rescored from the definition.  log Z and
    the gradients are compared with the oracle on the same recipe at T = 20 000
    (the float64 oracle needs about 13 minutes for the full length)."""
    w = wl.make_workload("stress")
    g = run_gpu(w)
    assert g["status"] == 0 and g["vstatus"] == 0
    L = int(w.lengths[0])
    dvec = np.arange(1, w.K + 1)[:, None]
    np.testing.assert_allclose((dvec * g["dD"]).sum(), L, rtol=1e-10)          # total length
    np.testing.assert_allclose(g["dD"].sum() - g["dA"].sum(), 1.0, atol=1e-5)   # segments - transitions
    np.testing.assert_allclose(g["dX"][0, :L].sum(axis=1), 0.0, atol=1e-4)     # coverage sums to one
    assert g["dA"].min() >= 0 and g["dD"].min() >= 0
    assert np.isfinite(g["logZ"]).all()
    # Viterbi: a valid segmentation whose score, recomputed from the definition,
    # is the returned score and does not exceed log Z
    seg = g["seg_start"][0, :L].astype(bool)
    assert seg[0]
    starts = np.flatnonzero(seg)
    assert np.diff(np.append(starts, L)).max() <= w.K
    s = oracle.path_score(w.x, w.A, w.D, w.lengths, g["labels"], g["seg_start"])
    np.testing.assert_allclose(g["score"], s, rtol=1e-11)
    assert g["score"][0] <= g["logZ"][0]
    # the same recipe, shorter: full parity with the oracle
    w2 = wl.make_workload("stress", T=20000)
    g2 = run_gpu(w2)
    lz = oracle.logz(w2.x, w2.A, w2.D, w2.lengths)
    assert g2["status"] == 0 and abs(g2["logZ"][0] - lz[0]) / abs(lz[0]) <= 1e-11



# ------------------------------------------------------------------ fused path
@pytest.mark.parametrize("name,path", [("tiny", None), ("ner", None), ("tiny", "general"), ("ner", "general")])
def test_fused_named_small(name, path, monkeypatch):
    if path:
        monkeypatch.setenv("SEMICRF_KERNEL_PATH", path)
    w = wl.make_workload(name)
    grad = np.linspace(0.5, 1.5, w.B)
    check_against_oracle(w, run_gpu_fused(w, grad=grad), grad=grad)


@pytest.mark.parametrize("seed,B,T,K,C", [(8, 9, 90, 32, 32), (1, 5, 100, 1, 7), (4, 1, 1, 4, 5),
                                           (5, 2, 50, 200, 9), (6, 3, 300, 40, 64), (7, 2, 200, 300, 20),
                                           (2, 2, 70, 70, 2), (3, 4, 129, 33, 33),
                                           # C, K <= 32: more items than post-pass CTAs; the longest
                                           # single-launch scan; past it (three-pass scan)
                                           (11, 40, 700, 16, 17), (12, 3, 1024, 32, 32), (13, 2, 2100, 8, 5),
                                           (14, 7, 33, 32, 1)])
def test_fused_random_shapes(seed, B, T, K, C):
    w = wl.random_small(seed, B, T, K, C, ragged=True)
    check_against_oracle(w, run_gpu_fused(w))


@pytest.mark.parametrize("path,K", [(None, 12), ("general", 12), (None, 160)])
def test_fused_rebased_columns(path, K, monkeypatch):
    # emissions of standard deviation 12: log Z grows by ~18 per position, so the
    # per-label references of both chains move every few dozen positions and the
    # passes over the stored rows take their exact-scaling branch (K = 160: the
    # dD contraction's 128-duration tile)
    if path:
        monkeypatch.setenv("SEMICRF_KERNEL_PATH", path)
    w = wl.random_small(15, 4, 400, K, 9, ragged=True, scale=12.0)
    grad = np.array([1.0, -0.5, 2.0, 0.25])
    check_against_oracle(w, run_gpu_fused(w, grad=grad), grad=grad)


@pytest.mark.parametrize("name", ["ner", "tiny"])
def test_host_buffer_step_equals_device_step(name):
    # semicrf_forward_backward_host: the same kernels on the same inputs, so the
    # same bits as prefix_scan + forward_backward on device tensors
    torch = _torch()
    import semi_markov_crf_prefix_b200 as sc
    w = wl.make_workload(name)
    grad = np.linspace(0.5, 1.5, w.B)
    g = run_gpu_fused(w, grad=grad)
    dev = torch.device("cuda:0")
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
    stage = sc.new_host_stage(w.B, w.T, w.K, w.C, device=dev)
    sc.clear_device_status(ws)
    logZ, dA, dD, dX = sc.forward_backward_host(pin(w.x), pin(w.A), pin(w.D), pin(w.lengths), ws, stage,
                                                grad_logZ=pin(grad), want_dX=True)
    assert sc.device_status(ws) == 0   # synchronises the stream
    for k, v in (("logZ", logZ), ("dA", dA), ("dD", dD), ("dX", dX)):
        assert np.array_equal(v.numpy(), g[k]), k


def test_fused_large_workloads():
    for w in (wl.make_workload("speech", B=4, T=1500), wl.make_workload("genomic", T=6000),
              wl.make_workload("large", B=2, T=1500)):
        check_against_oracle(w, run_gpu_fused(w))


def test_fused_equals_checkpointed_path():
    # the two ways of computing the same gradients agree to rounding
    for w in (wl.make_workload("ner", B=8), wl.random_small(44, 3, 200, 40, 48, ragged=True)):
        a, b = run_gpu(w), run_gpu_fused(w)
        np.testing.assert_allclose(a["logZ"], b["logZ"], rtol=1e-14)
        for k in ("dA", "dD"):
            np.testing.assert_allclose(a[k], b[k], atol=1e-9, rtol=1e-11)
        np.testing.assert_allclose(a["dX"], b["dX"], atol=2e-7, rtol=0)
