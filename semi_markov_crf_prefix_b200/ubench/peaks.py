"""Measured throughput of the units the chains are bound by (FP64 FMA, FP32 FMA,
MUFU ex2) on the GPU at hand, with the SM clock sampled during the run.

    python -m semi_markov_crf_prefix_b200.ubench.peaks     # prints one JSON line

``build()`` compiles ``peaks.cu`` (sm_100a) into the executable ``peaks`` next to
it; ``measure()`` runs it in its own process (its own CUDA context, so it leaves
the caller's untouched) and returns operations per second per unit, the median
SM clock under load and the per-SM-per-clock rates derived from it.
"""
from __future__ import annotations

import json
import os
import statistics
import subprocess
import sys
import threading
from pathlib import Path

HERE = Path(__file__).resolve().parent
SRC = HERE / "peaks.cu"
EXE = HERE / "peaks"


def build(force: bool = False) -> Path:
    if force or not EXE.exists() or EXE.stat().st_mtime < SRC.stat().st_mtime:
        nvcc = os.environ.get("NVCC") or "/usr/local/cuda/bin/nvcc"
        if not Path(nvcc).exists():
            nvcc = "nvcc"
        tmp = EXE.with_suffix(".tmp")
        subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
                        "-o", str(tmp), str(SRC)], check=True)
        os.replace(tmp, EXE)
    return EXE


def _sample_clocks(stop, out, gpu_index):
    try:
        p = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), "--query-gpu=clocks.sm,clocks.max.sm",
                              "--format=csv,noheader,nounits", "-lms", "50"],
                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
    except Exception:
        return
    try:
        while not stop.is_set():
            line = p.stdout.readline()
            if not line:
                break
            f = [v.strip() for v in line.split(",")]
            try:
                out.append((float(f[0]), float(f[1])))
            except (ValueError, IndexError):
                pass
    finally:
        p.terminate()
        try:
            p.wait(timeout=5)
        except Exception:
            p.kill()


def measure(reps: int = 10, gpu_index: int = 0) -> dict:
    exe = build()
    stop, samples = threading.Event(), []
    th = threading.Thread(target=_sample_clocks, args=(stop, samples, gpu_index), daemon=True)
    th.start()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES=os.environ.get("CUDA_VISIBLE_DEVICES", str(gpu_index)))
    r = subprocess.run([str(exe), str(reps)], capture_output=True, text=True, env=env, timeout=300)
    stop.set()
    th.join(timeout=10)
    if r.returncode != 0:
        raise RuntimeError(f"peaks microbenchmark failed: {r.stderr.strip()}")
    out = json.loads(r.stdout.strip().splitlines()[-1])
    # samples taken while a kernel ran: the clock under load (idle samples read lower or equal)
    loaded = [m for m, _ in samples]
    out["sm_mhz_median"] = statistics.median(loaded) if loaded else None
    out["sm_mhz_max"] = max(m for _, m in samples) if samples else None
    mhz = out["sm_mhz_median"]
    if mhz:
        hz = mhz * 1e6 * out["sms"]
        out["fp64_fma_per_sm_clk"] = out["fp64_fma_per_s"] / hz
        out["fp32_fma_per_sm_clk"] = out["fp32_fma_per_s"] / hz
        out["mufu_ex2_per_sm_clk"] = out["mufu_ex2_per_s"] / hz
    return out


if __name__ == "__main__":
    print(json.dumps(measure(int(sys.argv[1]) if len(sys.argv) > 1 else 10)))
