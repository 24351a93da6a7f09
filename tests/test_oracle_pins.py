"""Pins for the CPU oracle: each checks it against something other than itself.

Every test here runs on the CPU (no GPU).  The pins are chosen so that a
plausible slip anywhere in the oracle (a dropped term, a wrong sign or index, a
transposed transition) fails at least one of them:

  P1  brute-force enumeration of every segmentation (T = 10)
  P2  closed forms for all-zero scores (exact integer counts)
  P3  edge-potential tier (direct inner sums) == factorised tier
  P4  K = 1 reduces to a linear-chain CRF (dense matrix products, textbook Viterbi)
  P5  finite differences of log Z for every input
  P6  probabilistic invariants (coverage sums to one, counts, forward == backward)
  P7  centring semantics (duration-prior equivalence, invariance to per-label and
      per-position constants)
  P8  reversal symmetry
  P9  Viterbi: enumeration, path score recomputed from the definition, score <= log Z
  P10 segment-start probabilities: enumeration, all-zero closed form, expected
      number of segments
  P11 gold-path gradient: finite differences of the path score, feature counts
  M8  drift of the cumulative scores: centred << uncentred, S[L] = 0
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import bruteforce as bf
import semicrf_workloads as wl


@pytest.fixture(scope="module")
def tiny10():
    return wl.make_workload("tiny10")


@pytest.fixture(scope="module")
def tiny():
    return wl.make_workload("tiny")


@pytest.fixture(scope="module")
def ner():
    return wl.make_workload("ner")


# --------------------------------------------------------------------------- P1
def test_p1_bruteforce_tiny10(tiny10):
    w = tiny10
    e = bf.enumerate_batch(w.x, w.A, w.D, w.lengths)
    f = oracle.factorised(w.x, w.A, w.D, w.lengths, want_mu=True)
    d = oracle.edge_direct(w.x, w.A, w.D, w.lengths, want_mu=True)
    for r in (f, d):
        np.testing.assert_allclose(r["logZ"], e["logZ"], rtol=1e-12, atol=0)
        np.testing.assert_allclose(r["dA"], e["dA"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["dD"], e["dD"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["dX"], e["dX"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["mu"], e["mu"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["logZ_bwd"], e["logZ"], rtol=1e-12, atol=0)


def test_p1_bruteforce_ragged_small():
    # ragged lengths (including L = 1 and L < K), two label counts
    for seed, (B, T, K, C) in enumerate([(4, 8, 3, 3), (3, 7, 8, 2), (2, 9, 2, 4)]):
        w = wl.random_small(seed + 11, B, T, K, C, ragged=True)
        w.lengths[0] = 1
        e = bf.enumerate_batch(w.x, w.A, w.D, w.lengths)
        f = oracle.factorised(w.x, w.A, w.D, w.lengths)
        np.testing.assert_allclose(f["logZ"], e["logZ"], rtol=1e-12)
        np.testing.assert_allclose(f["dA"], e["dA"], atol=1e-12)
        np.testing.assert_allclose(f["dD"], e["dD"], atol=1e-12)
        np.testing.assert_allclose(f["dX"], e["dX"], atol=1e-12)
        # padding rows carry no gradient
        for b in range(B):
            assert np.all(f["dX"][b, w.lengths[b]:] == 0)


def test_p1_bruteforce_uncentred_and_weights(tiny10):
    w = tiny10
    g = np.array([0.75, -1.5])
    e = bf.enumerate_batch(w.x, w.A, w.D, w.lengths, centre=False)
    f = oracle.factorised(w.x, w.A, w.D, w.lengths, centre=False, grad_logZ=g)
    np.testing.assert_allclose(f["logZ"], e["logZ"], rtol=1e-12)
    # weighted gradients: sum_b g_b * (per-sequence gradient)
    per = [bf.enumerate_sequence(w.x[b], w.A, w.D, int(w.lengths[b]), centre=False)
           for b in range(2)]
    np.testing.assert_allclose(f["dA"], g[0] * per[0]["dA"] + g[1] * per[1]["dA"], atol=1e-12)
    np.testing.assert_allclose(f["dD"], g[0] * per[0]["dD"] + g[1] * per[1]["dD"], atol=1e-12)
    np.testing.assert_allclose(f["dX"][0, :10], g[0] * per[0]["dX"], atol=1e-12)
    np.testing.assert_allclose(f["dX"][1, :10], g[1] * per[1]["dX"], atol=1e-12)


def test_bruteforce_counts_segmentations():
    # the enumeration itself: C*(1+C)**(L-1) labelled segmentations when K >= L
    for L, C in [(1, 3), (4, 2), (6, 3)]:
        assert bf.count_segmentations(L, L, C) == C * (1 + C) ** (L - 1)


# --------------------------------------------------------------------------- P2
def _zero_counts(L, K, C):
    """Exact number of labelled segmentations of [0, L) with durations <= K."""
    N = [1] + [0] * L
    for t in range(1, L + 1):
        N[t] = C * sum(N[t - d] for d in range(1, min(K, t) + 1))
    return N[L]


@pytest.mark.parametrize("L,K,C", [(7, 7, 3), (12, 20, 4), (30, 4, 5), (50, 1, 3), (64, 8, 4)])
def test_p2_zero_scores_closed_form(L, K, C):
    x = np.zeros((1, L, C))
    A = np.zeros((C, C))
    D = np.zeros((K, C))
    lengths = np.array([L], np.int32)
    f = oracle.factorised(x, A, D, lengths)
    d = oracle.edge_direct(x, A, D, lengths) if L <= 30 else None
    expect = math.log(_zero_counts(L, K, C))
    if K >= L:
        assert _zero_counts(L, K, C) == C * (1 + C) ** (L - 1)
    np.testing.assert_allclose(f["logZ"][0], expect, rtol=1e-13)
    if d is not None:
        np.testing.assert_allclose(d["logZ"][0], expect, rtol=1e-13)
    if K >= L:
        # every interior boundary is present with probability C/(1+C), labels uniform
        nseg = 1 + (L - 1) * C / (1 + C)
        np.testing.assert_allclose(f["dD"].sum(), nseg, rtol=1e-12)
        np.testing.assert_allclose(f["dA"], np.full((C, C), (L - 1) / (C * (1 + C))), rtol=1e-11)
        # coverage is uniform over labels
        np.testing.assert_allclose(f["dX"], 0.0, atol=1e-13)


def _golden_zero_scores():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "zero_scores.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    return [(int(L), int(K), int(C), float(z)) for L, K, C, z in rows]


def test_p2_golden_zero_scores_fixture():
    # the stored closed-form values (exact integer counts) against the oracle,
    # at the shapes the oracle finishes quickly
    rows = _golden_zero_scores()
    assert len(rows) >= 4
    for L, K, C, z in rows:
        if L * (K * C + C * C) > 2e7:
            continue
        assert math.isclose(math.log(_zero_counts(L, K, C)), z, rel_tol=1e-15)
        f = oracle.factorised(np.zeros((1, L, C)), np.zeros((C, C)), np.zeros((K, C)), np.array([L], np.int32))
        np.testing.assert_allclose(f["logZ"][0], z, rtol=1e-13)


def test_p2_viterbi_tie_break_on_zeros():
    # all candidates tie: smallest d (=1) each time, smallest previous label (0),
    # final label 0  ->  every position a segment of label 0
    L, K, C = 9, 4, 3
    x = np.zeros((1, L, C))
    score, labels, seg = oracle.viterbi(x, np.zeros((C, C)), np.zeros((K, C)), np.array([L]))
    assert score[0] == 0.0
    assert np.all(labels[0] == 0)
    assert np.all(seg[0] == 1)


# --------------------------------------------------------------------------- P3
def test_p3_edge_direct_equals_factorised_tiny(tiny):
    w = tiny
    f = oracle.factorised(w.x, w.A, w.D, w.lengths, want_mu=True)
    d = oracle.edge_direct(w.x, w.A, w.D, w.lengths, want_mu=True)
    np.testing.assert_allclose(d["logZ"], f["logZ"], rtol=1e-11)
    for k in ("dX", "dA", "dD", "mu"):
        np.testing.assert_allclose(d[k], f[k], atol=1e-11, err_msg=k)


def test_p3_edge_direct_equals_factorised_ner(ner):
    w = ner
    f = oracle.factorised(w.x, w.A, w.D, w.lengths)
    d = oracle.edge_direct(w.x, w.A, w.D, w.lengths)
    np.testing.assert_allclose(d["logZ"], f["logZ"], rtol=1e-11)
    np.testing.assert_allclose(d["dX"], f["dX"], atol=1e-10)
    np.testing.assert_allclose(d["dA"], f["dA"], atol=1e-9, rtol=1e-11)
    np.testing.assert_allclose(d["dD"], f["dD"], atol=1e-9, rtol=1e-11)


# --------------------------------------------------------------------------- P4
def _linear_chain(xc, Dd0, A):
    """Textbook linear-chain CRF on unary x - nu + D[0]: scaled matrix products."""
    L, C = xc.shape
    phi = np.exp(xc + Dd0[None, :])
    EA = np.exp(A)
    alpha = phi[0].copy()
    log_scale = 0.0
    alphas = [alpha / alpha.sum()]
    scales = [math.log(alpha.sum())]
    for t in range(1, L):
        alpha = (alphas[-1] @ EA) * phi[t]
        s = alpha.sum()
        alphas.append(alpha / s)
        scales.append(math.log(s))
    logZ = sum(scales)
    beta = np.ones(C)
    betas = [beta]
    for t in range(L - 1, 0, -1):
        beta = EA @ (phi[t] * betas[0])
        beta = beta / beta.sum()
        betas.insert(0, beta)
    mu = np.array([a * b for a, b in zip(alphas, betas)])
    mu /= mu.sum(axis=1, keepdims=True)
    del log_scale
    return logZ, mu


def _linear_viterbi(xc, Dd0, A):
    L, C = xc.shape
    u = xc + Dd0[None, :]
    v = u[0].copy()
    back = np.zeros((L, C), np.int64)
    for t in range(1, L):
        cand = v[:, None] + A            # [prev, cur]
        back[t] = np.argmax(cand, axis=0)
        v = cand.max(axis=0) + u[t]
    path = [int(np.argmax(v))]
    for t in range(L - 1, 0, -1):
        path.insert(0, int(back[t, path[0]]))
    return float(v.max()), np.array(path)


def test_p4_linear_chain_reduction():
    for seed, (B, T, C) in enumerate([(3, 40, 5), (2, 200, 7)]):
        w = wl.random_small(100 + seed, B, T, 1, C, ragged=True)
        f = oracle.factorised(w.x, w.A, w.D, w.lengths, want_mu=True)
        s, labels, seg = oracle.viterbi(w.x, w.A, w.D, w.lengths)
        for b in range(B):
            L = int(w.lengths[b])
            x = w.x[b, :L].astype(np.float64)
            xc = x - x.mean(axis=0)
            logZ, mu = _linear_chain(xc, w.D[0].astype(np.float64), w.A.astype(np.float64))
            np.testing.assert_allclose(f["logZ"][b], logZ, rtol=1e-12)
            np.testing.assert_allclose(f["mu"][b, :L], mu, atol=1e-12)
            vs, vp = _linear_viterbi(xc, w.D[0].astype(np.float64), w.A.astype(np.float64))
            np.testing.assert_allclose(s[b], vs, rtol=1e-12)
            assert np.array_equal(labels[b, :L], vp)
            assert np.all(seg[b, :L] == 1)


# --------------------------------------------------------------------------- P5
def _fd(fun, theta, h=2.0 ** -12, indices=None):
    """Central differences with exact (float64) step sizes; theta is modified in place."""
    assert theta.flags.c_contiguous
    flat = theta.reshape(-1)
    idx = range(flat.size) if indices is None else indices
    out = np.empty(len(idx))
    for j, i in enumerate(idx):
        old = flat[i]
        step = h * max(1.0, abs(old))
        flat[i] = old + step
        fp = fun()
        flat[i] = old - step
        fm = fun()
        flat[i] = old
        out[j] = (fp - fm) / (2 * step)
    return out if indices is not None else out.reshape(theta.shape)


def test_p5_finite_differences_tiny(tiny):
    w = tiny
    x = w.x.astype(np.float64).copy()
    A = w.A.astype(np.float64).copy()
    D = w.D.astype(np.float64).copy()
    g = np.array([1.0, -0.5])
    f = oracle.factorised(x, A, D, w.lengths, grad_logZ=g)

    def obj():
        return float(np.dot(g, oracle.logz(x, A, D, w.lengths, nthreads=1)))

    np.testing.assert_allclose(_fd(obj, A), f["dA"], atol=1e-7)
    np.testing.assert_allclose(_fd(obj, D), f["dD"], atol=1e-7)
    np.testing.assert_allclose(_fd(obj, x), f["dX"], atol=1e-7)


def test_p5_finite_differences_detached_nu(tiny):
    # With nu held fixed the x-gradient is the coverage alone: it equals the
    # gradient of the uncentred model evaluated at x - nu, checked by differences.
    w = tiny
    S, nu = oracle.prefix(w.x, w.lengths)
    xc = np.ascontiguousarray(w.x.astype(np.float64) - nu[:, None, :])
    f = oracle.factorised(w.x, w.A, w.D, w.lengths, detach_nu=True)
    u = oracle.factorised(xc, w.A, w.D, w.lengths, centre=False)
    np.testing.assert_allclose(f["dX"], u["dX"], atol=1e-12)
    A = w.A.astype(np.float64)
    D = w.D.astype(np.float64)

    def obj():
        return float(oracle.logz(xc, A, D, w.lengths, centre=False, nthreads=1).sum())

    idx = np.random.default_rng(3).choice(xc.size, 64, replace=False)
    fd = _fd(obj, xc, indices=idx)
    np.testing.assert_allclose(fd, u["dX"].reshape(-1)[idx], atol=1e-7)
    # and the centred gradient differs from it by the per-label mean of coverage
    assert np.abs(f["dX"] - oracle.factorised(w.x, w.A, w.D, w.lengths)["dX"]).max() > 1e-3


# --------------------------------------------------------------------------- P6
def test_p6_invariants_ner(ner):
    w = ner
    f = oracle.factorised(w.x, w.A, w.D, w.lengths, want_mu=True)
    mu = f["mu"]
    for b in range(w.B):
        L = int(w.lengths[b])
        np.testing.assert_allclose(mu[b, :L].sum(axis=1), 1.0, atol=1e-12)      # I1
        assert mu[b].min() >= -1e-12 and mu[b].max() <= 1 + 1e-12                # I2
        np.testing.assert_allclose(f["dX"][b].sum(axis=0), 0.0, atol=1e-10)      # I3
    K = w.K
    dvec = np.arange(1, K + 1)[:, None]
    np.testing.assert_allclose((dvec * f["dD"]).sum(), w.lengths.sum(), rtol=1e-12)   # I4
    np.testing.assert_allclose(f["dD"].sum() - f["dA"].sum(), w.B, rtol=1e-12)        # I5
    np.testing.assert_allclose(f["logZ_bwd"], f["logZ"], rtol=1e-13)                  # I6
    assert f["dA"].min() >= 0 and f["dD"].min() >= 0


# --------------------------------------------------------------------------- P7
def test_p7_centring_is_a_duration_prior(tiny):
    # logZ(x; A, D) == logZ_uncentred(x; A, D - d*nu), one sequence at a time
    w = tiny
    S, nu = oracle.prefix(w.x, w.lengths)
    f = oracle.logz(w.x, w.A, w.D, w.lengths)
    for b in range(w.B):
        d = np.arange(1, w.K + 1, dtype=np.float64)[:, None]
        Db = w.D.astype(np.float64) - d * nu[b][None, :]
        u = oracle.logz(w.x[b:b + 1], w.A, Db, w.lengths[b:b + 1], centre=False)
        np.testing.assert_allclose(u[0], f[b], rtol=1e-13)


def test_p7_invariance_to_constants(ner):
    w = ner
    rng = np.random.default_rng(5)
    f = oracle.factorised(w.x, w.A, w.D, w.lengths)
    kappa = rng.normal(0, 3, size=(w.B, 1, w.C))          # per (b, c) constant
    g = oracle.factorised(w.x + kappa, w.A, w.D, w.lengths)
    np.testing.assert_allclose(g["logZ"], f["logZ"], rtol=1e-12)
    np.testing.assert_allclose(g["dX"], f["dX"], atol=1e-10)
    lam = rng.normal(0, 3, size=(w.B, w.T, 1))            # per-position constant
    h = oracle.factorised(w.x + lam, w.A, w.D, w.lengths)
    np.testing.assert_allclose(h["logZ"], f["logZ"], rtol=1e-12)
    np.testing.assert_allclose(h["dX"], f["dX"], atol=1e-10)
    # without centring the per-label constant is not absorbed
    u0 = oracle.logz(w.x, w.A, w.D, w.lengths, centre=False)
    u1 = oracle.logz(w.x + kappa, w.A, w.D, w.lengths, centre=False)
    assert np.abs(u1 - u0).max() > 1.0


# --------------------------------------------------------------------------- P8
def test_p8_reversal_symmetry(ner):
    w = ner
    f = oracle.logz(w.x, w.A, w.D, w.lengths)
    xr = np.zeros_like(w.x)
    for b in range(w.B):
        L = int(w.lengths[b])
        xr[b, :L] = w.x[b, :L][::-1]
    r = oracle.logz(xr, w.A.T.copy(), w.D, w.lengths)
    np.testing.assert_allclose(r, f, rtol=1e-12)
    # a non-symmetric A matters: without the transpose the value changes
    r2 = oracle.logz(xr, w.A, w.D, w.lengths)
    assert np.abs(r2 - f).max() > 1e-3


# --------------------------------------------------------------------------- P9
def test_p9_viterbi(tiny10, tiny, ner):
    w = tiny10
    e = bf.enumerate_batch(w.x, w.A, w.D, w.lengths)
    s, labels, seg = oracle.viterbi(w.x, w.A, w.D, w.lengths)
    np.testing.assert_allclose(s, e["score"], rtol=1e-12)
    assert np.array_equal(labels, e["labels"])
    assert np.array_equal(seg, e["seg_start"])
    for w in (tiny, ner):
        s, labels, seg = oracle.viterbi(w.x, w.A, w.D, w.lengths)
        ps = oracle.path_score(w.x, w.A, w.D, w.lengths, labels, seg)
        np.testing.assert_allclose(ps, s, rtol=1e-11)
        lz = oracle.logz(w.x, w.A, w.D, w.lengths)
        assert np.all(s <= lz)
        for b in range(w.B):
            L = int(w.lengths[b])
            assert np.all(labels[b, L:] == -1) and np.all(seg[b, L:] == 0)
            assert seg[b, 0] == 1 and np.all(labels[b, :L] >= 0)
            # segment durations respect K
            starts = np.flatnonzero(seg[b, :L])
            assert np.diff(np.append(starts, L)).max() <= w.K


def test_p9_same_label_duration_swap_is_an_exact_tie(ner):
    # Two adjacent segments of one label score the same in either order of their
    # durations: the emission sums telescope to the same span and the same D and A
    # terms appear.  So the best segmentation is not unique wherever it holds such
    # a pair (the labels per position still are): brute force on a tiny problem
    # finds several argmax segmentations with equal labels, and the definition
    # scores the swapped segmentations of NER's Viterbi paths equal to rounding.
    w = wl.random_small(3, 1, 6, 6, 1, ragged=False)   # one label: only durations differ
    best, ties = -np.inf, []
    for durs in bf.compositions(6, 6):
        starts = np.zeros((1, 6), np.uint8)
        starts[0, np.cumsum((0,) + durs[:-1])] = 1
        sc = oracle.path_score(w.x, w.A, w.D, w.lengths, np.zeros((1, 6), np.int32), starts)[0]
        if sc > best + 1e-12:
            best, ties = sc, [starts]
        elif abs(sc - best) <= 1e-12:
            ties.append(starts)
    durs = [tuple(np.diff(np.append(np.flatnonzero(t[0]), 6))) for t in ties]
    assert all(sorted(d) == sorted(durs[0]) for d in durs)
    assert len(ties) == math.factorial(len(durs[0])) // math.prod(
        math.factorial(durs[0].count(v)) for v in set(durs[0]))
    s, labels, seg = oracle.viterbi(ner.x, ner.A, ner.D, ner.lengths)
    swapped = 0
    for b in range(ner.B):
        L = int(ner.lengths[b])
        starts = list(np.flatnonzero(seg[b, :L])) + [L]
        for i in range(len(starts) - 2):
            a, m, e = starts[i], starts[i + 1], starts[i + 2]
            if labels[b, a] == labels[b, m] and (m - a) != (e - m):
                alt = seg.copy()
                alt[b, m] = 0
                alt[b, a + (e - m)] = 1
                ps = oracle.path_score(ner.x[b:b + 1], ner.A, ner.D, ner.lengths[b:b + 1],
                                       labels[b:b + 1], alt[b:b + 1])[0]
                assert abs(ps - s[b]) <= 1e-12 * abs(s[b])
                swapped += 1
    assert swapped > 0


# --------------------------------------------------------------------------- M8
def test_m8_centring_controls_drift(ner):
    w = ner
    Sc, nu = oracle.prefix(w.x, w.lengths, centre=True)
    Su, _ = oracle.prefix(w.x, w.lengths, centre=False)
    assert np.abs(Sc).max() * 5 < np.abs(Su).max()
    for b in range(w.B):
        L = int(w.lengths[b])
        np.testing.assert_allclose(Sc[b, L], 0.0, atol=1e-10)
        assert np.all(Sc[b, L:] == Sc[b, L])
    for b in range(w.B):
        L = int(w.lengths[b])
        np.testing.assert_allclose(nu[b], w.x[b, :L].astype(np.float64).mean(axis=0), rtol=1e-12)


# -------------------------------------------------------------------------- P10
def test_p10_start_probabilities_bruteforce(tiny10):
    w = tiny10
    e = bf.enumerate_batch(w.x, w.A, w.D, w.lengths)
    f = oracle.factorised(w.x, w.A, w.D, w.lengths, want_pstart=True)
    np.testing.assert_allclose(f["pstart"], e["pstart"], rtol=0, atol=1e-12)
    # a ragged batch: zero beyond L_b, one at 0
    w2 = wl.random_small(seed=31, B=3, T=9, K=4, C=3, ragged=True)
    e2 = bf.enumerate_batch(w2.x, w2.A, w2.D, w2.lengths)
    f2 = oracle.factorised(w2.x, w2.A, w2.D, w2.lengths, want_pstart=True)
    np.testing.assert_allclose(f2["pstart"], e2["pstart"], rtol=0, atol=1e-12)
    for b in range(w2.B):
        assert f2["pstart"][b, 0] == pytest.approx(1.0, abs=1e-13)
        assert np.all(f2["pstart"][b, w2.lengths[b]:] == 0.0)


@pytest.mark.parametrize("L,K,C", [(7, 7, 3), (12, 20, 4)])
def test_p10_start_probabilities_zero_scores(L, K, C):
    # all-zero scores with K >= L: each interior boundary independently present
    # with probability C / (1 + C)
    f = oracle.factorised(np.zeros((1, L, C)), np.zeros((C, C)), np.zeros((K, C)),
                          np.array([L], np.int32), want_pstart=True)
    expect = np.full(L, C / (1 + C))
    expect[0] = 1.0
    np.testing.assert_allclose(f["pstart"][0], expect, rtol=1e-12)


def test_p10_expected_segment_count(ner):
    # each segment has exactly one start: sum_s P(start at s) = E[#segments] = sum dD
    w = wl.make_workload("ner", B=4, T=128)
    f = oracle.factorised(w.x, w.A, w.D, w.lengths, want_pstart=True)
    for b in range(w.B):
        fb = oracle.factorised(w.x[b:b + 1], w.A, w.D, w.lengths[b:b + 1])
        np.testing.assert_allclose(f["pstart"][b].sum(), fb["dD"].sum(), rtol=1e-12)


# -------------------------------------------------------------------------- P11
def _random_segmentation(rng, L, K, C, T):
    labels = np.full(T, -1, np.int32)
    seg = np.zeros(T, np.uint8)
    s = 0
    while s < L:
        d = int(rng.integers(1, min(K, L - s) + 1))
        c = int(rng.integers(0, C))
        labels[s:s + d] = c
        seg[s] = 1
        s += d
    return labels, seg


def test_p11_path_gradient_finite_differences(tiny):
    w = tiny
    rng = np.random.default_rng(5)
    labels = np.zeros((w.B, w.T), np.int32)
    seg = np.zeros((w.B, w.T), np.uint8)
    for b in range(w.B):
        labels[b], seg[b] = _random_segmentation(rng, int(w.lengths[b]), w.K, w.C, w.T)
    g = np.array([0.7, -1.3])
    dX, dA, dD = oracle.path_grads(w.x, w.A, w.D, w.lengths, labels, seg, grad=g)

    def f(x, A, D):
        return float(np.dot(g, oracle.path_score(x, A, D, w.lengths, labels, seg)))

    x0, A0, D0 = (np.asarray(v, np.float64).copy() for v in (w.x, w.A, w.D))
    h = 1e-3   # the score is linear: central differences are exact up to rounding
    for (arr, grad) in ((x0, dX), (A0, dA), (D0, dD)):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = arr[i]
            arr[i] = old + h
            fp = f(x0, A0, D0)
            arr[i] = old - h
            fm = f(x0, A0, D0)
            arr[i] = old
            num[i] = (fp - fm) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=0, atol=1e-9)


def test_p11_path_counts(ner):
    w = wl.make_workload("ner", B=3, T=100)
    rng = np.random.default_rng(9)
    labels = np.zeros((w.B, w.T), np.int32)
    seg = np.zeros((w.B, w.T), np.uint8)
    for b in range(w.B):
        labels[b], seg[b] = _random_segmentation(rng, int(w.lengths[b]), w.K, w.C, w.T)
    dX, dA, dD = oracle.path_grads(w.x, w.A, w.D, w.lengths, labels, seg)
    nseg = int(seg.sum())
    assert dD.sum() == pytest.approx(nseg)
    assert dA.sum() == pytest.approx(nseg - w.B)
    assert (np.arange(1, w.K + 1)[:, None] * dD).sum() == pytest.approx(int(w.lengths.sum()))
    np.testing.assert_allclose(dX.sum(axis=1), 0.0, atol=1e-12)   # centring: zero sum over positions


def test_long_sequence_forward_backward_agree():
    """Forward and backward log Z of a long sequence agree to two ulps of log Z:
    the messages are kept relative to exact integer offsets, so the rounding of
    each position does not accumulate with the magnitude of log Z (~5e4 here);
    without the offsets the two drift 26 ulps (1.9e-10) apart at this length,
    and ~2e-8 apart at the large-label workload's 2e5 positions."""
    w = wl.make_workload("large", B=1, T=20000, K=24, C=8)
    o = oracle.factorised(w.x, w.A, w.D, w.lengths, nthreads=1)
    lz, lzb = float(o["logZ"][0]), float(o["logZ_bwd"][0])
    assert abs(lz) > 5e4
    assert abs(lz - lzb) <= 2 * np.spacing(abs(lz)), (lz, lzb)
    # the marginals still sum to one per position at this length
    L = int(w.lengths[0])
    dvec = np.arange(1, w.K + 1)[:, None]
    np.testing.assert_allclose((dvec * o["dD"]).sum(), L, rtol=1e-12)
