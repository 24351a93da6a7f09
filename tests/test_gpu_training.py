"""GPU parity for the outputs around the hot path: posterior marginals (coverage
and segment-start probabilities), the score of gold segmentations and its
gradient, and the negative log-likelihood as a torch.autograd.Function.  All
against the float64 CPU oracle; the posterior outputs are float32, so they are
held to 1e-6 absolute."""
import numpy as np
import pytest

import oracle
import semicrf_workloads as wl

pytestmark = pytest.mark.gpu

POST_ATOL = 1e-6
GRAD_ATOL = 1e-4


def _dev(w):
    import torch
    dev = torch.device("cuda:0")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return dev, t(w.x), t(w.A), t(w.D), t(w.lengths)


def _random_segmentations(w, seed):
    rng = np.random.default_rng(seed)
    labels = np.full((w.B, w.T), -1, np.int32)
    seg = np.zeros((w.B, w.T), np.uint8)
    for b in range(w.B):
        L, s = int(w.lengths[b]), 0
        while s < L:
            d = int(rng.integers(1, min(w.K, L - s) + 1))
            labels[b, s:s + d] = int(rng.integers(0, w.C))
            seg[b, s] = 1
            s += d
    return labels, seg


def _posteriors(w, path=None, monkeypatch=None):
    import semi_markov_crf_prefix_b200 as sc
    if path and monkeypatch:
        monkeypatch.setenv("SEMICRF_KERNEL_PATH", path)
    dev, x, A, D, lens = _dev(w)
    ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
    sc.clear_device_status(ws)
    S, _ = sc.prefix_scan(x, lens, ws=ws)
    sc.forward(S, A, D, lens, ws=ws)
    mu, ps = sc.posteriors(S, A, D, lens, ws)
    assert sc.device_status(ws) == 0
    return mu.cpu().numpy(), ps.cpu().numpy()


@pytest.mark.parametrize("name,path", [("tiny", None), ("ner", None), ("ner", "general"), ("tiny", "general")])
def test_posteriors_match_oracle(name, path, monkeypatch):
    w = wl.make_workload(name)
    mu, ps = _posteriors(w, path, monkeypatch)
    o = oracle.factorised(w.x, w.A, w.D, w.lengths, want_mu=True, want_pstart=True)
    np.testing.assert_allclose(mu, o["mu"], rtol=0, atol=POST_ATOL)
    np.testing.assert_allclose(ps, o["pstart"], rtol=0, atol=POST_ATOL)
    for b in range(w.B):
        L = int(w.lengths[b])
        np.testing.assert_allclose(mu[b, :L].sum(axis=-1), 1.0, atol=1e-5)   # every position covered once
        assert np.all(mu[b, L:] == 0.0) and np.all(ps[b, L:] == 0.0)


def test_posteriors_cluster_shape():
    # a shape only the cluster kernels take (C > 32), ragged lengths
    w = wl.random_small(seed=41, B=3, T=160, K=40, C=48, ragged=True)
    mu, ps = _posteriors(w)
    o = oracle.factorised(w.x, w.A, w.D, w.lengths, want_mu=True, want_pstart=True)
    np.testing.assert_allclose(mu, o["mu"], rtol=0, atol=POST_ATOL)
    np.testing.assert_allclose(ps, o["pstart"], rtol=0, atol=POST_ATOL)


@pytest.mark.parametrize("name", ["tiny", "ner"])
def test_gold_score_and_gradient(name):
    import torch
    import semi_markov_crf_prefix_b200 as sc
    w = wl.make_workload(name)
    labels, seg = _random_segmentations(w, seed=3)
    dev, x, A, D, lens = _dev(w)
    tl = torch.from_numpy(labels).to(dev)
    tsg = torch.from_numpy(seg).to(dev)
    ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
    sc.clear_device_status(ws)
    S, _ = sc.prefix_scan(x, lens, ws=ws)
    score = sc.gold_score(S, A, D, lens, tl, tsg, ws).cpu().numpy()
    g = np.linspace(-1.0, 2.0, w.B)
    dX = torch.zeros((w.B, w.T, w.C), dtype=torch.float32, device=dev)
    dA = torch.zeros((w.C, w.C), dtype=torch.float64, device=dev)
    dD = torch.zeros((w.K, w.C), dtype=torch.float64, device=dev)
    sc.gold_backward(lens, tl, tsg, ws, dX, dA, dD, grad_score=torch.from_numpy(g).to(dev))
    assert sc.device_status(ws) == 0
    np.testing.assert_allclose(score, oracle.path_score(w.x, w.A, w.D, w.lengths, labels, seg), rtol=1e-12)
    eX, eA, eD = oracle.path_grads(w.x, w.A, w.D, w.lengths, labels, seg, grad=g)
    np.testing.assert_allclose(dX.cpu().numpy(), eX, rtol=0, atol=1e-6)
    np.testing.assert_allclose(dA.cpu().numpy(), eA, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dD.cpu().numpy(), eD, rtol=0, atol=1e-12)


def test_gold_score_of_viterbi_path():
    # the Viterbi path scored by the gold kernel equals the Viterbi score
    import semi_markov_crf_prefix_b200 as sc
    w = wl.make_workload("ner")
    dev, x, A, D, lens = _dev(w)
    ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
    S, _ = sc.prefix_scan(x, lens, ws=ws)
    vs, vl, vg = sc.viterbi(S, A, D, lens)
    score = sc.gold_score(S, A, D, lens, vl, vg, ws)
    assert sc.device_status(ws) == 0
    np.testing.assert_allclose(score.cpu().numpy(), vs.cpu().numpy(), rtol=1e-12, atol=1e-9)


@pytest.mark.parametrize("name,path", [("ner", None), ("ner", "general")])
def test_nll_autograd(name, path, monkeypatch):
    import torch
    import semi_markov_crf_prefix_b200 as sc
    if path:
        monkeypatch.setenv("SEMICRF_KERNEL_PATH", path)
    w = wl.make_workload(name, B=8)
    labels, seg = _random_segmentations(w, seed=11)
    dev, x, A, D, lens = _dev(w)
    x.requires_grad_(True)
    A.requires_grad_(True)
    D.requires_grad_(True)
    nll = sc.semicrf_nll(x, A, D, lens, torch.from_numpy(labels).to(dev), torch.from_numpy(seg).to(dev))
    g = torch.linspace(0.5, 1.5, w.B, dtype=torch.float64, device=dev)
    (nll * g).sum().backward()
    o = oracle.factorised(w.x, w.A, w.D, w.lengths, grad_logZ=g.cpu().numpy())
    ps = oracle.path_score(w.x, w.A, w.D, w.lengths, labels, seg)
    pX, pA, pD = oracle.path_grads(w.x, w.A, w.D, w.lengths, labels, seg, grad=g.cpu().numpy())
    np.testing.assert_allclose(nll.detach().cpu().numpy(), o["logZ"] - ps, rtol=1e-9, atol=1e-8)
    assert np.all(nll.detach().cpu().numpy() >= -1e-9)   # log Z >= score of any segmentation
    np.testing.assert_allclose(x.grad.cpu().numpy(), o["dX"] - pX, rtol=0, atol=GRAD_ATOL)
    np.testing.assert_allclose(A.grad.cpu().numpy(), o["dA"] - pA, rtol=0, atol=GRAD_ATOL)
    np.testing.assert_allclose(D.grad.cpu().numpy(), o["dD"] - pD, rtol=0, atol=GRAD_ATOL)


def test_gold_malformed_segmentation_reports_status():
    # errors made on the host: a segmentation that does not start at 0, one longer
    # than K, one whose label changes inside a segment, a label out of range
    import torch
    import semi_markov_crf_prefix_b200 as sc
    w = wl.make_workload("tiny")
    dev, x, A, D, lens = _dev(w)
    labels, seg = _random_segmentations(w, seed=1)
    bad = []
    s0 = seg.copy(); s0[0, 0] = 0; s0[0, 1] = 1; bad.append((labels, s0))
    s1 = np.zeros_like(seg); s1[:, 0] = 1; l1 = np.zeros_like(labels); bad.append((l1, s1))   # one segment of length T > K
    l2 = labels.copy()
    s = next(s for s in range(int(w.lengths[1]) - 1) if seg[1, s] and not seg[1, s + 1])
    l2[1, s + 1] = (l2[1, s] + 1) % w.C   # label changes inside a segment
    bad.append((l2, seg))
    l3 = labels.copy(); l3[0, 0] = w.C; bad.append((l3, seg))
    for lb, sg in bad:
        ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
        sc.clear_device_status(ws)
        S, _ = sc.prefix_scan(x, lens, ws=ws)
        sc.gold_score(S, A, D, lens, torch.from_numpy(lb).to(dev), torch.from_numpy(sg).to(dev), ws)
        assert sc.device_status(ws) == sc._lib.SEMICRF_ERR_INVALID_SEGMENTATION


def test_nll_entry_points():
    # semicrf_nll forms log Z - score on the device from the same log Z and score
    # the separate calls give; semicrf_nll_backward equals the backward with
    # weights g followed by the gold backward with weights -g
    import torch
    import semi_markov_crf_prefix_b200 as sc
    w = wl.make_workload("ner", B=6)
    labels, seg = _random_segmentations(w, seed=5)
    dev, x, A, D, lens = _dev(w)
    lb, sg = torch.from_numpy(labels).to(dev), torch.from_numpy(seg).to(dev)
    g = torch.linspace(-1.0, 2.0, w.B, dtype=torch.float64, device=dev)
    ws = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
    sc.clear_device_status(ws)
    S, _ = sc.prefix_scan(x, lens, ws=ws)
    nll, logZ, score = sc.nll(S, A, D, lens, lb, sg, ws)
    dX, dA, dD = sc.nll_backward(S, A, D, lens, lb, sg, ws, grad_nll=g)
    assert sc.device_status(ws) == 0
    ws2 = sc.new_workspace(w.B, w.T, w.K, w.C, sc.WS_TRAIN, device=dev)
    sc.clear_device_status(ws2)
    logZ2, _ = sc.forward(S, A, D, lens, ws=ws2)
    score2 = sc.gold_score(S, A, D, lens, lb, sg, ws2)
    rX, rA, rD = sc.backward(S, A, D, lens, ws2, grad_logZ=g)
    sc.gold_backward(lens, lb, sg, ws2, rX, rA, rD, grad_score=(-g).contiguous())
    assert sc.device_status(ws2) == 0
    assert torch.equal(logZ, logZ2) and torch.equal(score, score2)
    assert torch.equal(nll, logZ2 - score2)
    for a, b in ((dX, rX), (dA, rA), (dD, rD)):
        assert torch.equal(a, b)
