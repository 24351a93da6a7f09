"""Stored float64 oracle results for the full-size workloads (test data).

The factorised oracle takes hours of CPU on the large-label workload
(B=4, T=200 000, K=512, C=256) and minutes on the genomic one, so the full-size
parity tests read its results from files written by this script, which calls
only ``oracle/`` and the seeded input generator.  Nothing here comes from the
CUDA path.

    python tests/oracle_cache.py large genomic stress50k [--threads N]

Each entry is ``tests/_oracle_cache/<name>-seed<seed>-<key>.npz`` where the key
is a hash of the oracle's C source, its Python wrapper and the input generator,
so a change to any of them makes the tests ignore a stale file.  Contents:
log Z [B], dA [C,C], dD [K,C] (float64, g = 1), the Viterbi score [B], labels
[B,T] and segment starts [B,T], and dX at the positions listed in ``dx_pos``
(every position for the smaller workloads; for the large-label workload every
128th position plus the first and last 256 of each sequence, which is 17 MB
instead of 1.6 GB).

The large-label workload is run one sequence at a time (the per-sequence
gradients summed in sequence order afterwards, exactly as the oracle sums them)
so that an interrupted run keeps the sequences it finished.
"""
from __future__ import annotations

import argparse
import hashlib
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import semicrf_workloads as wl  # noqa: E402

CACHE_DIR = os.path.join(HERE, "_oracle_cache")

# name -> (workload recipe, B, T); None keeps the recipe's own size
ENTRIES = {
    "large": ("large", None, None),
    "genomic": ("genomic", None, None),
    "stress50k": ("stress", 1, 50_000),
}


def key() -> str:
    h = hashlib.sha256()
    for rel in ("oracle/semicrf_oracle.c", "oracle/__init__.py", "semicrf_workloads.py"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def path(name: str, seed: int = 0) -> str:
    return os.path.join(CACHE_DIR, f"{name}-seed{seed}-{key()}.npz")


def workload(name: str, seed: int = 0):
    recipe, B, T = ENTRIES[name]
    return wl.make_workload(recipe, seed=seed, B=B, T=T)


def dx_positions(name: str, T: int) -> np.ndarray:
    if name != "large":
        return np.arange(T, dtype=np.int64)
    pos = set(range(0, T, 128)) | set(range(256)) | set(range(T - 256, T))
    return np.array(sorted(pos), dtype=np.int64)


def load(name: str, seed: int = 0):
    """The stored result as a dict, or None when it has not been written."""
    p = path(name, seed)
    if not os.path.exists(p):
        return None
    with np.load(p) as z:
        return {k: z[k] for k in z.files}


def _partial(name, seed, b):
    return os.path.join(CACHE_DIR, f"{name}-seed{seed}-{key()}.b{b}.npz")


def build(name: str, seed: int = 0, threads: int = 0, log=print) -> str:
    import oracle
    oracle.build()
    w = workload(name, seed)
    pos = dx_positions(name, w.T)
    os.makedirs(CACHE_DIR, exist_ok=True)
    parts = []
    for b in range(w.B):
        pp = _partial(name, seed, b)
        if not os.path.exists(pp):
            t0 = time.time()
            sl = slice(b, b + 1)
            r = oracle.factorised(w.x[sl], w.A, w.D, w.lengths[sl], nthreads=threads)
            score, labels, seg = oracle.viterbi(w.x[sl], w.A, w.D, w.lengths[sl], nthreads=threads)
            tmp = pp + ".tmp.npz"
            np.savez(tmp, logZ=r["logZ"], logZ_bwd=r["logZ_bwd"], dA=r["dA"], dD=r["dD"],
                     dX=r["dX"][0][pos], score=score, labels=labels, seg_start=seg)
            os.replace(tmp, pp)
            log(f"{name} b={b}: {time.time() - t0:.0f} s")
        with np.load(pp) as z:
            parts.append({k: z[k] for k in z.files})
    # per-sequence gradients summed in sequence order from zero, as the oracle does for g = 1
    dA = np.zeros_like(parts[0]["dA"])
    dD = np.zeros_like(parts[0]["dD"])
    for p in parts:
        dA += p["dA"]
        dD += p["dD"]
    out = dict(
        logZ=np.concatenate([p["logZ"] for p in parts]),
        logZ_bwd=np.concatenate([p["logZ_bwd"] for p in parts]),
        dA=dA, dD=dD, dx_pos=pos,
        dX=np.stack([p["dX"] for p in parts]),
        score=np.concatenate([p["score"] for p in parts]),
        labels=np.concatenate([p["labels"] for p in parts]),
        seg_start=np.concatenate([p["seg_start"] for p in parts]),
    )
    final = path(name, seed)
    tmp = final + ".tmp.npz"
    np.savez(tmp, **out)
    os.replace(tmp, final)
    for b in range(w.B):
        os.remove(_partial(name, seed, b))
    return final


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("names", nargs="+", choices=sorted(ENTRIES))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--threads", type=int, default=0)
    args = ap.parse_args()
    for n in args.names:
        if load(n, args.seed) is not None:
            print(f"{n}: present ({path(n, args.seed)})")
            continue
        print(f"{n}: wrote {build(n, args.seed, args.threads)}", flush=True)


if __name__ == "__main__":
    main()
