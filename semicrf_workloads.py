"""Seeded synthetic semi-CRF workloads (host-side, numpy only).

This module only draws inputs.  It holds none of the semi-CRF arithmetic, so the
CPU oracle (``oracle/``) and the CUDA path can both be fed from it without sharing
any of the method's code.

Every workload is drawn with ``numpy.random.Generator(PCG64(seed))`` in a fixed
order: emissions x, then transitions A, then duration bias D, then lengths or
segment structure.  Emissions are float32 ``[B, T, C]`` (label fastest),
transitions float32 ``[C, C]`` indexed ``[from, to]``, duration bias float32
``[K, C]`` with row ``d-1`` for duration d, lengths int32 ``[B]``.

The shapes and value distributions stand in for the workloads named on the
Flash-SemiCRF pages (named-entity tagging, phoneme segmentation of speech,
genomic segmentation at T = 100 000, and a large-label long-sequence stress
case).  The pages give no data; nothing here is a dataset item.

Readings of the distribution recipe (standard deviations throughout):
  * "N(0, s)" is a normal with standard deviation s.
  * speech: a width-5 moving average centred on t, averaged over the positions
    that exist (the window shrinks at both ends).
  * genomic: segments with geometric lengths (support 1, 2, ..., mean 200),
    labels i.i.d. uniform, drawn until they cover T; +1.5 on the segment's
    own label only.
  * large: a per-label mean offset 2 * (c + 1) ** -1.1 (Zipf exponent 1.1,
    amplitude 2 so that label 0 matches the +2 "outside" offset of the
    named-entity workload).
  * stress: the scale test of one million positions with K = 200 (the pages'
    scalability claim); C = 24 and the genomic recipe (geometric segments of
    mean 200 with +1.5 on the true label) are this module's choice.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = ["Workload", "CONFIGS", "make_workload", "config_dims"]


@dataclass
class Workload:
    name: str
    B: int
    T: int
    K: int
    C: int
    x: np.ndarray        # float32 [B, T, C]
    A: np.ndarray        # float32 [C, C]  (from, to)
    D: np.ndarray        # float32 [K, C]  (row d-1)
    lengths: np.ndarray  # int32 [B], each in [1, T]
    seed: int

    @property
    def updates(self) -> int:
        """B*T*K*C: the segment-label update count the throughput metric uses."""
        return self.B * self.T * self.K * self.C

    @property
    def valid_updates(self) -> int:
        """sum_b L_b*K*C: the work actually present on ragged lengths."""
        return int(self.lengths.astype(np.int64).sum()) * self.K * self.C


# name -> (B, T, K, C)
CONFIGS = {
    "tiny": (2, 64, 8, 4),
    "tiny10": (2, 10, 8, 4),
    "ner": (32, 512, 16, 17),
    "speech": (16, 4000, 64, 128),
    "genomic": (1, 100_000, 1000, 24),
    "large": (4, 200_000, 512, 256),
    "stress": (1, 1_000_000, 200, 24),
}


def config_dims(name: str):
    return CONFIGS[name]


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _normal32(rng, shape, std=1.0):
    out = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def _tiny(name, B, T, K, C, seed):
    rng = _rng(seed)
    x = _normal32(rng, (B, T, C))
    A = _normal32(rng, (C, C), 0.1)
    D = _normal32(rng, (K, C), 0.1)
    lengths = np.full(B, T, dtype=np.int32)
    return Workload(name, B, T, K, C, x, A, D, lengths, seed)


def _ner(B, T, K, C, seed):
    rng = _rng(seed)
    x = _normal32(rng, (B, T, C))
    x[:, :, 0] += np.float32(2.0)          # the "outside" label is over-represented
    A = _normal32(rng, (C, C), 0.5)
    D = _normal32(rng, (K, C), 0.5)
    lengths = rng.integers(T // 2, T + 1, size=B).astype(np.int32)
    return Workload("ner", B, T, K, C, x, A, D, lengths, seed)


def _speech(B, T, K, C, seed):
    rng = _rng(seed)
    raw = rng.standard_normal((B, T, C), dtype=np.float32).astype(np.float64)
    # centred width-5 moving average over the positions that exist
    csum = np.concatenate([np.zeros((B, 1, C)), np.cumsum(raw, axis=1)], axis=1)
    t = np.arange(T)
    lo = np.maximum(t - 2, 0)
    hi = np.minimum(t + 3, T)
    x = np.ascontiguousarray(((csum[:, hi, :] - csum[:, lo, :]) / (hi - lo)[None, :, None]).astype(np.float32))
    A = _normal32(rng, (C, C), 0.3)
    d = np.arange(1, K + 1, dtype=np.float32)[:, None]
    D = (np.float32(-0.05) * d + _normal32(rng, (K, C), 0.1)).astype(np.float32)
    lengths = np.full(B, T, dtype=np.int32)
    return Workload("speech", B, T, K, C, x, A, D, lengths, seed)


def genomic_segments(rng, T, C, mean_len=200.0):
    """Geometric segment lengths (support >= 1) with uniform labels covering T."""
    starts, labels = [], []
    t = 0
    while t < T:
        n = int(rng.geometric(1.0 / mean_len))
        starts.append(t)
        labels.append(int(rng.integers(0, C)))
        t += n
    return np.array(starts, dtype=np.int64), np.array(labels, dtype=np.int64)


def _genomic(B, T, K, C, seed, mean_len=200.0, name="genomic"):
    rng = _rng(seed)
    x = _normal32(rng, (B, T, C))
    A = _normal32(rng, (C, C), 0.3)
    D = _normal32(rng, (K, C), 0.1)
    for b in range(B):
        starts, labels = genomic_segments(rng, T, C, mean_len)
        ends = np.append(starts[1:], T)
        for s, e, c in zip(starts, ends, labels):
            x[b, s:e, c] += np.float32(1.5)
    lengths = np.full(B, T, dtype=np.int32)
    return Workload(name, B, T, K, C, x, A, D, lengths, seed)


def _large(B, T, K, C, seed):
    rng = _rng(seed)
    x = _normal32(rng, (B, T, C))
    offs = (2.0 * (np.arange(C, dtype=np.float64) + 1.0) ** -1.1).astype(np.float32)
    x += offs[None, None, :]
    A = _normal32(rng, (C, C), 0.2)
    D = _normal32(rng, (K, C), 0.1)
    lengths = np.full(B, T, dtype=np.int32)
    return Workload("large", B, T, K, C, x, A, D, lengths, seed)


def make_workload(name: str, seed: int = 0, *, B=None, T=None, K=None, C=None) -> Workload:
    """Draw a named workload; B/T/K/C override the named shape (same recipe).

    ``T`` shorter than the named one keeps the recipe (for the named-entity
    workload the lengths are drawn in [T/2, T]).
    """
    B0, T0, K0, C0 = CONFIGS[name]
    B = B0 if B is None else B
    T = T0 if T is None else T
    K = K0 if K is None else K
    C = C0 if C is None else C
    if name in ("tiny", "tiny10"):
        return _tiny(name, B, T, K, C, seed)
    if name == "ner":
        return _ner(B, T, K, C, seed)
    if name == "speech":
        return _speech(B, T, K, C, seed)
    if name == "genomic":
        return _genomic(B, T, K, C, seed)
    if name == "large":
        return _large(B, T, K, C, seed)
    if name == "stress":
        return _genomic(B, T, K, C, seed, name="stress")
    raise KeyError(name)


def random_small(seed: int, B: int, T: int, K: int, C: int, ragged: bool = True,
                 scale: float = 1.0) -> Workload:
    """Small random problem for sweeps (ragged lengths in [1, T] when asked)."""
    rng = _rng(seed)
    x = _normal32(rng, (B, T, C), scale)
    A = _normal32(rng, (C, C), 0.5)
    D = _normal32(rng, (K, C), 0.5)
    if ragged:
        lengths = rng.integers(1, T + 1, size=B).astype(np.int32)
    else:
        lengths = np.full(B, T, dtype=np.int32)
    return Workload("random", B, T, K, C, x, A, D, lengths, seed)
