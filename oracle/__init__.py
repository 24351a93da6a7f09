"""Plain float64 CPU semi-CRF oracle.  TEST INFRASTRUCTURE ONLY.

The checker for the CUDA path.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  It shares no code with
the CUDA library and never imports it.

Functions here marshal numpy arrays (widened to float64; float32 data widens
exactly) into ``liboracle.so`` (plain C, built from
``semicrf_oracle.c`` by :func:`build`).  Every formula lives in the C source, which
cites the passage of the Flash-SemiCRF pages each step follows.  The brute-force
enumeration tier is pure Python/numpy in :mod:`oracle.bruteforce`.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "semicrf_oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (-O2, OpenMP, no FP contraction)."""
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(".so.tmp")
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               "-o", str(tmp), str(_SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB_PATH))
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_prefix.argtypes = [i, i, i, P, P, i, P, P]
        lib.oracle_factorised.argtypes = [i, i, i, i, P, P, P, P, i, i, P, P, P, P, P, P, P, P, i]
        lib.oracle_logz.argtypes = [i, i, i, i, P, P, P, P, i, P, i]
        lib.oracle_edge_direct.argtypes = [i, i, i, i, P, P, P, P, i, i, P, P, P, P, P, P, i]
        lib.oracle_viterbi.argtypes = [i, i, i, i, P, P, P, P, i, P, P, P, i]
        for f in (lib.oracle_prefix, lib.oracle_factorised, lib.oracle_logz,
                  lib.oracle_edge_direct, lib.oracle_viterbi):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _prep(x, A, D, lengths):
    x = np.ascontiguousarray(x, dtype=np.float64)
    A = np.ascontiguousarray(A, dtype=np.float64)
    D = np.ascontiguousarray(D, dtype=np.float64)
    lengths = np.ascontiguousarray(lengths, dtype=np.int32)
    B, T, C = x.shape
    K = D.shape[0]
    assert A.shape == (C, C) and D.shape == (K, C) and lengths.shape == (B,)
    return x, A, D, lengths, B, T, K, C


def _check(rc):
    if rc != 0:
        raise ValueError("oracle: invalid lengths (each must lie in [1, T])")


def prefix(x, lengths, centre=True):
    """nu [B,C] and S [B,T+1,C] (float64)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    lengths = np.ascontiguousarray(lengths, dtype=np.int32)
    B, T, C = x.shape
    S = np.empty((B, T + 1, C), np.float64)
    nu = np.empty((B, C), np.float64)
    _check(_load().oracle_prefix(B, T, C, _p(x), _p(lengths), int(centre), _p(S), _p(nu)))
    return S, nu


def factorised(x, A, D, lengths, centre=True, detach_nu=False, grad_logZ=None,
               want_mu=False, want_pstart=False, nthreads=0):
    """log Z, backward log Z, dX, dA, dD (and coverage mu, start probability
    pstart) from the factorised tier."""
    x, A, D, lengths, B, T, K, C = _prep(x, A, D, lengths)
    g = None if grad_logZ is None else np.ascontiguousarray(grad_logZ, dtype=np.float64)
    logZ = np.empty(B, np.float64)
    logZ_bwd = np.empty(B, np.float64)
    dX = np.empty((B, T, C), np.float64)
    dA = np.empty((C, C), np.float64)
    dD = np.empty((K, C), np.float64)
    mu = np.empty((B, T, C), np.float64) if want_mu else None
    ps = np.empty((B, T), np.float64) if want_pstart else None
    _check(_load().oracle_factorised(B, T, K, C, _p(x), _p(A), _p(D), _p(lengths), int(centre),
                                     int(detach_nu), _p(g), _p(logZ), _p(logZ_bwd), _p(dX),
                                     _p(dA), _p(dD), _p(mu), _p(ps), int(nthreads)))
    out = dict(logZ=logZ, logZ_bwd=logZ_bwd, dX=dX, dA=dA, dD=dD)
    if want_mu:
        out["mu"] = mu
    if want_pstart:
        out["pstart"] = ps
    return out


def logz(x, A, D, lengths, centre=True, nthreads=0):
    """Forward-only log Z [B] (factorised recursion)."""
    x, A, D, lengths, B, T, K, C = _prep(x, A, D, lengths)
    out = np.empty(B, np.float64)
    _check(_load().oracle_logz(B, T, K, C, _p(x), _p(A), _p(D), _p(lengths), int(centre),
                               _p(out), int(nthreads)))
    return out


def edge_direct(x, A, D, lengths, centre=True, detach_nu=False, grad_logZ=None,
                want_mu=False, nthreads=0):
    """log Z, dX, dA, dD (and mu) from the edge-potential tier (small sizes)."""
    x, A, D, lengths, B, T, K, C = _prep(x, A, D, lengths)
    g = None if grad_logZ is None else np.ascontiguousarray(grad_logZ, dtype=np.float64)
    logZ = np.empty(B, np.float64)
    dX = np.empty((B, T, C), np.float64)
    dA = np.empty((C, C), np.float64)
    dD = np.empty((K, C), np.float64)
    mu = np.empty((B, T, C), np.float64) if want_mu else None
    _check(_load().oracle_edge_direct(B, T, K, C, _p(x), _p(A), _p(D), _p(lengths), int(centre),
                                      int(detach_nu), _p(g), _p(logZ), _p(dX), _p(dA), _p(dD),
                                      _p(mu), int(nthreads)))
    out = dict(logZ=logZ, dX=dX, dA=dA, dD=dD)
    if want_mu:
        out["mu"] = mu
    return out


def viterbi(x, A, D, lengths, centre=True, nthreads=0):
    """score [B] float64, labels [B,T] int32 (-1 past L_b), seg_start [B,T] uint8."""
    x, A, D, lengths, B, T, K, C = _prep(x, A, D, lengths)
    score = np.empty(B, np.float64)
    labels = np.empty((B, T), np.int32)
    seg_start = np.empty((B, T), np.uint8)
    _check(_load().oracle_viterbi(B, T, K, C, _p(x), _p(A), _p(D), _p(lengths), int(centre),
                                  _p(score), _p(labels), _p(seg_start), int(nthreads)))
    return score, labels, seg_start


def path_grads(x, A, D, lengths, labels, seg_start, centre=True, grad=None):
    """Gradient of sum_b g_b path_score_b with respect to x, A, D, from the
    definition: the score is linear in x (through the segment sums and nu), in A
    (one term per transition) and in D (one term per segment)."""
    x = np.asarray(x, np.float64)
    B, T, C = x.shape
    K = np.asarray(D).shape[0]
    dX = np.zeros((B, T, C))
    dA = np.zeros((C, C))
    dD = np.zeros((K, C))
    for b in range(B):
        g = 1.0 if grad is None else float(grad[b])
        L = int(lengths[b])
        starts = [s for s in range(L) if seg_start[b, s]]
        ends = starts[1:] + [L]
        prev = None
        for s, e in zip(starts, ends):
            c = int(labels[b, s])
            dX[b, s:e, c] += g                    # d/dx of sum_{u=s}^{e-1} x[u,c]
            if centre:
                dX[b, :L, c] -= g * (e - s) / L   # d/dx of -(e-s) nu[c], nu = mean over u < L
            dD[e - s - 1, c] += g
            if prev is not None:
                dA[prev, c] += g
            prev = c
    return dX, dA, dD


def path_score(x, A, D, lengths, labels, seg_start, centre=True):
    """Score of a given segmentation, summed from the definition (direct sums)."""
    x = np.asarray(x, np.float64)
    A = np.asarray(A, np.float64)
    D = np.asarray(D, np.float64)
    B = x.shape[0]
    out = np.empty(B)
    for b in range(B):
        L = int(lengths[b])
        nu = x[b, :L].mean(axis=0) if centre else np.zeros(x.shape[2])
        starts = [s for s in range(L) if seg_start[b, s]]
        ends = starts[1:] + [L]
        total, prev = 0.0, None
        for s, e in zip(starts, ends):
            c = int(labels[b, s])
            total += float((x[b, s:e, c] - nu[c]).sum()) + float(D[e - s - 1, c])
            if prev is not None:
                total += float(A[prev, c])
            prev = c
        out[b] = total
    return out
