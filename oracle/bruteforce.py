"""Brute-force enumeration tier of the oracle.  TEST INFRASTRUCTURE ONLY.

Enumerates every segmentation of [0, L) with durations 1..K and every label
sequence, scores each from the definition (direct sums of centred emissions,
duration bias, transitions between consecutive segments; Streaming Structured
Inference with Flash-SemiCRF, abstract and technical summary section 1) and
returns log Z, its exact gradients (expected feature counts) and the best
segmentation.  Cost is about C*(1+C)**(L-1) scores, so only tiny inputs
(L <= 10, C <= 4) are practical.

Labels of one composition (d_1..d_n) are enumerated at once as an n-dimensional
numpy grid, one axis per segment.
"""
from __future__ import annotations

import numpy as np


def compositions(L: int, K: int):
    """All tuples (d_1, ..., d_n) of integers in [1, K] summing to L."""
    if L == 0:
        yield ()
        return
    for d in range(1, min(K, L) + 1):
        for rest in compositions(L - d, K):
            yield (d,) + rest


def _score_grid(xc, A, D, durs):
    """Scores of all label sequences for one composition, shape (C,)*n."""
    C = xc.shape[1]
    n = len(durs)
    grid = np.zeros((C,) * n)
    s = 0
    for i, d in enumerate(durs):
        unary = xc[s:s + d].sum(axis=0) + D[d - 1]
        shape = [1] * n
        shape[i] = C
        grid = grid + unary.reshape(shape)
        if i >= 1:
            shape2 = [1] * n
            shape2[i - 1] = C
            shape2[i] = C
            grid = grid + A.reshape(shape2)
        s += d
    return grid


def enumerate_sequence(x, A, D, L, centre=True):
    """Exact quantities for one sequence by enumeration.

    x: [T, C] (only the first L rows are used).  Returns dict with logZ, dA [C,C],
    dD [K,C], mu [L,C] (coverage), pstart [L] (probability that a segment
    begins at each position), dX [L,C] (gradient w.r.t. x, including the
    path through the centring baseline when centre is set), best (score,
    list of (s, d, c)).
    """
    x = np.asarray(x, np.float64)[:L]
    A = np.asarray(A, np.float64)
    D = np.asarray(D, np.float64)
    K, C = D.shape
    nu = x.mean(axis=0) if centre else np.zeros(C)
    xc = x - nu
    comps = list(compositions(L, K))
    # pass 1: log Z and best path
    m = -np.inf
    parts = []
    best = (-np.inf, None)
    for durs in comps:
        g = _score_grid(xc, A, D, durs)
        gm = g.max()
        parts.append((gm, np.exp(g - gm).sum()))
        if gm > best[0]:
            idx = np.unravel_index(int(np.argmax(g)), g.shape)
            best = (float(gm), (durs, idx))
        m = max(m, gm)
    logZ = m + np.log(sum(s * np.exp(gm - m) for gm, s in parts))
    # pass 2: expected counts
    dA = np.zeros((C, C))
    dD = np.zeros((K, C))
    mu = np.zeros((L, C))
    pstart = np.zeros(L)
    for durs in comps:
        n = len(durs)
        P = np.exp(_score_grid(xc, A, D, durs) - logZ)
        total = P.sum()        # probability of this set of boundaries (all labellings)
        s = 0
        for d in durs:
            pstart[s] += total
            s += d
        s = 0
        for i, d in enumerate(durs):
            axes = tuple(j for j in range(n) if j != i)
            marg = P.sum(axis=axes) if axes else P
            dD[d - 1] += marg
            mu[s:s + d] += marg[None, :]
            if i >= 1:
                axes2 = tuple(j for j in range(n) if j not in (i - 1, i))
                pair = P.sum(axis=axes2) if axes2 else P
                dA += pair
            s += d
    dX = mu - (mu.mean(axis=0, keepdims=True) if centre else 0.0)
    durs, labs = best[1]
    segs = []
    s = 0
    for d, c in zip(durs, labs):
        segs.append((s, d, int(c)))
        s += d
    return dict(logZ=float(logZ), dA=dA, dD=dD, mu=mu, pstart=pstart, dX=dX, best_score=best[0],
                best_segs=segs)


def enumerate_batch(x, A, D, lengths, centre=True):
    """Batch version: logZ [B], dX [B,T,C], dA, dD summed over the batch, best paths."""
    x = np.asarray(x, np.float64)
    B, T, C = x.shape
    K = np.asarray(D).shape[0]
    logZ = np.empty(B)
    dX = np.zeros((B, T, C))
    mu = np.zeros((B, T, C))
    pstart = np.zeros((B, T))
    dA = np.zeros((C, C))
    dD = np.zeros((K, C))
    scores = np.empty(B)
    labels = np.full((B, T), -1, np.int32)
    seg_start = np.zeros((B, T), np.uint8)
    for b in range(B):
        L = int(lengths[b])
        r = enumerate_sequence(x[b], A, D, L, centre)
        logZ[b] = r["logZ"]
        dX[b, :L] = r["dX"]
        mu[b, :L] = r["mu"]
        pstart[b, :L] = r["pstart"]
        dA += r["dA"]
        dD += r["dD"]
        scores[b] = r["best_score"]
        for s, d, c in r["best_segs"]:
            labels[b, s:s + d] = c
            seg_start[b, s] = 1
    return dict(logZ=logZ, dX=dX, mu=mu, pstart=pstart, dA=dA, dD=dD, score=scores, labels=labels,
                seg_start=seg_start)


def count_segmentations(L: int, K: int, C: int) -> int:
    """Number of labelled segmentations, sum over compositions of C**n."""
    return sum(C ** len(c) for c in compositions(L, K))


__all__ = ["compositions", "enumerate_sequence", "enumerate_batch", "count_segmentations"]
