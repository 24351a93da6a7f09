"""bench.py host logic that needs no GPU: the reference arm's JSON line, the
algorithmic work counts, and the recorded DRAM traffic that must go stale when
the kernel source it was measured on changes."""
import json
import os
import shutil
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import semicrf_workloads as wl  # noqa: E402


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--steps", "1", "--warmup", "0", "--cpu-budget", "0.5"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = [l for l in out.stdout.splitlines() if l.startswith("{")][-1]
    d = json.loads(line)
    assert d["impl"] == "reference" and d["unit"] == "updates/s" and d["value"] > 0
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True and d["steps"] == 1
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


def test_algorithmic_counts():
    w = wl.make_workload("ner")
    sumL, terms, nbytes = bench.algorithmic(w)
    assert sumL == int(w.lengths.sum())
    assert terms == sumL * (w.K * w.C + w.C * w.C)
    assert nbytes == 8 * w.B * w.T * w.C + 8 * (w.C * w.C + w.K * w.C)


def test_recorded_traffic_goes_stale_with_the_source(tmp_path, monkeypatch):
    line = next(l for l in open(os.path.join(ROOT, "profiles", "dram_traffic.txt")).read().splitlines()
                if l.strip() and not l.startswith("#"))
    kernel, workload, nbytes, src, _ = line.split()
    assert bench.recorded_traffic(kernel, workload) == int(nbytes)
    # a copy of the repository view in which the kernel source differs by one byte
    (tmp_path / "profiles").mkdir()
    shutil.copy(os.path.join(ROOT, "profiles", "dram_traffic.txt"), tmp_path / "profiles" / "dram_traffic.txt")
    os.makedirs(tmp_path / os.path.dirname(src), exist_ok=True)
    data = open(os.path.join(ROOT, src), "rb").read()
    (tmp_path / src).write_bytes(data + b"\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic(kernel, workload) is None
    (tmp_path / src).write_bytes(data)
    assert bench.recorded_traffic(kernel, workload) == int(nbytes)
    assert bench.recorded_traffic(kernel, "no-such-workload") is None
