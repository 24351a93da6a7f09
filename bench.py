"""Benchmark: semi-CRF forward+backward throughput on B200.

One step = the whole hot path on one batch of synthetic input: centring and
prefix scan, then the forward and backward passes with exact gradients.  Two
ways to run the passes are timed:

  fused  semicrf_forward_backward: the forward chain (log Z, its per-position
         rows) and the backward chain side by side in one launch, then the
         marginal, coverage and gradient passes over the stored rows;
  ckpt   semicrf_forward + semicrf_backward: the checkpointed streaming pair
         (normalised checkpoints every ceil(sqrt(T)) positions, recompute of the
         segments in the backward).

The metric is B*T*K*C segment-label updates per second (whole job over all
ranks).  The headline line is the fused step on the large-label workload
(B=4, T=200 000, K=512, C=256); the same JSON line carries the checkpointed
pair on that workload (``paths``), every other named workload (``per_config``),
the roofline of the dominant kernel against unit peaks measured in the same run
(``roofline``, ``unit_peaks``), the end-to-end figure through the host-buffer
entry point (``e2e``) and the CPU oracle on a bounded sample (``cpu_baseline``).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config large] [--path fused|ckpt]
    python bench.py --impl reference ...   # the CPU oracle, same metric

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch (weak
scaling) and the parameter gradients dA, dD are summed across ranks with an
NCCL all-reduce inside the step.  Timing is CUDA events on the launching stream,
max over ranks; L2 is flushed (256 MiB write) between timed steps.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import semicrf_workloads as wl  # noqa: E402

METRIC = "semi-CRF fwd+bwd segment-label updates/sec (B·T·K·C/s), 1×B200, % roofline"
UNIT = "updates/s"
# B200 unit counts for the derived peaks: 148 SMs; per SM per clock 64 FP64 FMA
# lanes, 128 FP32 FMA lanes, 16 MUFU (special-function) lanes
N_SM = 148
FP64_FMA_PER_SM_CLK = 64
MUFU_PER_SM_CLK = 16
HBM_FALLBACK_GBS = 6650.0
SM_MAX_MHZ_FALLBACK = 1965.0
# every kernel one step launches, in launch order, keyed by the launch count the
# library reports for each call
SCAN_NAMES = {1: ["prefix_scan"], 3: ["scan_partials", "scan_offsets", "scan_apply"]}
FB_NAMES = {4: ["exp_tables", "chains", "post_rows", "post_finalise"],
            11: ["exp_tables", "chains", "rows_rescale", "cov_delta", "cov_offsets", "cov_scan", "cov_musum",
                 "dur_grad", "trans_grad", "finalise_params", "finalise_dx"]}
FWD_NAMES = {2: ["exp_tables", "fwd_chain"]}
BWD_NAMES = {4: ["recompute", "bwd_chain", "finalise_params", "finalise_dx"],
             6: ["recompute", "bwd_chain", "dur_grad", "trans_grad", "finalise_params", "finalise_dx"]}
PER_CONFIG = ["tiny", "ner", "speech", "genomic", "large", "stress"]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return json.load(f)
    except Exception:
        return None


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the last ncu capture of this kernel (profiles/
    dram_traffic.txt), or None when the kernel source changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    for line in lines:
        f = line.split()
        if len(f) != 5 or line.startswith("#") or f[0] != kernel or f[1] != workload:
            continue
        try:
            src = open(os.path.join(ROOT, f[3]), "rb").read()
        except OSError:
            return None
        return int(f[2]) if hashlib.sha256(src).hexdigest()[:16] == f[4] else None
    return None


def algorithmic(w):
    """Terms and bytes the method must do (not the recompute it chooses to do)."""
    sumL = int(w.lengths.astype(np.int64).sum())
    terms_pass = sumL * (w.K * w.C + w.C * w.C)          # one (lse,+) term = one FMA in exp space
    bytes_path = 4 * w.B * w.T * w.C * 2 + 8 * (w.C * w.C + w.K * w.C)
    return sumL, terms_pass, bytes_path


def roofline_times(w, peaks, hbm_gbs):
    """The workload's own bounds in ms: HBM bytes at the copy bandwidth, one MUFU
    exp per term (log space) and one FP64 FMA per term (exp space), at the unit
    rates given (operations per second)."""
    _, terms_pass, bytes_path = algorithmic(w)
    terms = 2 * terms_pass   # the forward and the backward pass
    return {"t_hbm_ms": bytes_path / (hbm_gbs * 1e9) * 1e3,
            "t_sfu_ms": terms / peaks["mufu_ex2_per_s"] * 1e3,
            "t_fp64_ms": terms / peaks["fp64_fma_per_s"] * 1e3}


def derived_unit_peaks(sm_mhz):
    hz = N_SM * sm_mhz * 1e6
    return {"fp64_fma_per_s": FP64_FMA_PER_SM_CLK * hz, "fp32_fma_per_s": 128 * hz,
            "mufu_ex2_per_s": MUFU_PER_SM_CLK * hz, "sm_mhz_median": sm_mhz,
            "source": f"derived: {N_SM} SMs x (64 FP64 FMA, 128 FP32 FMA, 16 MUFU) per clock x {sm_mhz:.0f} MHz"}


def live_unit_peaks(gpu_index):
    """FP64 FMA, FP32 FMA and MUFU ex2 rates measured now on this GPU
    (semi_markov_crf_prefix_b200/ubench/peaks.cu), or None if it cannot run."""
    try:
        from semi_markov_crf_prefix_b200.ubench import peaks
        out = peaks.measure(reps=10, gpu_index=gpu_index)
        out["source"] = ("measured live: semi_markov_crf_prefix_b200/ubench/peaks.cu, 148x8 CTAs x 256 threads "
                         "x 8 independent chains, best of 10 launches")
        return out
    except Exception as e:  # noqa: BLE001
        sys.stderr.write(f"unit-peak microbenchmark unavailable: {e}\n")
        return None


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        q = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)
        mhz, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9 or (self.uuid and f[0] != self.uuid):
                continue
            try:
                mhz.append(float(f[1]))
                maxes.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(mhz)}


# --------------------------------------------------------------------------- CPU oracle
def oracle_sample(w, budget_s=10.0, nthreads=0):
    """Time the CPU oracle (forward + backward + gradients) on a bounded sample of
    the workload: whole sequences, or a prefix of them when one is too slow."""
    import oracle
    nth = nthreads or os.cpu_count() or 1
    # estimate: ~4 log-space exponentials per term, ~1.5e7 per second per thread
    sumL, terms, _ = algorithmic(w)
    est = 4 * terms / (1.5e7 * nth)
    B, T = w.B, w.T
    x, lengths = w.x, w.lengths
    if est > budget_s:
        # shrink: fewer sequences, then a shorter prefix of each
        frac = budget_s / est
        Bs = max(1, min(B, int(math.ceil(B * frac))))
        Ts = T
        if Bs == 1 and frac * B < 1:
            Ts = max(w.K + 1, int(T * frac * B))
        x = np.ascontiguousarray(w.x[:Bs, :Ts])
        lengths = np.minimum(w.lengths[:Bs], Ts).astype(np.int32)
        B, T = Bs, Ts
    sample = f"B={B} of {w.B}, T={T} of {w.T}, K={w.K}, C={w.C}"
    oracle.build()
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.factorised(x, w.A, w.D, lengths, nthreads=nth)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 1000:
            break
    units = reps * B * T * w.K * w.C
    return {"value": units / el, "unit": UNIT, "cores": nth, "kind": "oracle",
            "sample": f"{sample}; {reps} repetition(s) in {el:.1f} s, float64 log-space, OpenMP; "
                      f"updates/s = B*T*K*C of the sample x repetitions / seconds"}


# --------------------------------------------------------------------------- GPU arm
def ctypes_void_p_array(n):
    import ctypes
    return ctypes.c_void_p * n


def ctypes_offset(arr, k):
    import ctypes
    return ctypes.cast(ctypes.byref(arr, k * ctypes.sizeof(ctypes.c_void_p)), ctypes.POINTER(ctypes.c_void_p))


class Runner:
    """Device buffers and one step of a path on one workload; per-kernel events."""

    def __init__(self, w, dev, path, ckpt=0, reduce_fn=None):
        import torch
        import semi_markov_crf_prefix_b200 as sc
        from semi_markov_crf_prefix_b200 import _lib
        self.torch, self.sc, self.w, self.path, self.ckpt = torch, sc, w, path, ckpt
        self.reduce_fn = reduce_fn
        B, T, K, C = w.B, w.T, w.K, w.C
        self.stream = torch.cuda.current_stream(dev)
        self.x = torch.from_numpy(w.x).to(dev)
        self.A = torch.from_numpy(w.A).to(dev)
        self.D = torch.from_numpy(w.D).to(dev)
        self.lens = torch.from_numpy(w.lengths).to(dev)
        self.ws = sc.new_workspace(B, T, K, C, sc.WS_TRAIN, ckpt, device=dev)
        self.S = torch.empty((B, T + 1, C), dtype=torch.float64, device=dev)
        self.nu = torch.empty((B, C), dtype=torch.float64, device=dev)
        self.logZ = torch.empty(B, dtype=torch.float64, device=dev)
        self.dX = torch.empty((B, T, C), dtype=torch.float32, device=dev)
        self.dA = torch.empty((C, C), dtype=torch.float64, device=dev)
        self.dD = torch.empty((K, C), dtype=torch.float64, device=dev)
        self.lib = _lib.load()
        # one untimed step to learn which kernels each call launches
        self.calls = self._calls()
        groups = []
        for fn, table in self.calls:
            fn()
            groups.append(table[sc.last_launch_count()])
        self.groups = groups
        self.names = [n for g in groups for n in g]
        self.evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(self.names))]
        for e in self.evs:
            e.record(self.stream)
        self.handles = (ctypes_void_p_array(len(self.evs)))(*[e.cuda_event for e in self.evs])

    def _calls(self):
        sc = self.sc
        scan = (lambda: sc.prefix_scan(self.x, self.lens, ws=self.ws, S=self.S, nu=self.nu), SCAN_NAMES)
        if self.path == "fused":
            return [scan, (lambda: sc.forward_backward(self.S, self.A, self.D, self.lens, ws=self.ws, logZ=self.logZ,
                                                       dX=self.dX, dA=self.dA, dD=self.dD), FB_NAMES)]
        return [scan,
                (lambda: sc.forward(self.S, self.A, self.D, self.lens, ws=self.ws, ckpt_interval=self.ckpt,
                                    logZ=self.logZ), FWD_NAMES),
                (lambda: sc.backward(self.S, self.A, self.D, self.lens, self.ws, ckpt_interval=self.ckpt,
                                     dX=self.dX, dA=self.dA, dD=self.dD), BWD_NAMES)]

    def step(self, profile=False):
        off = 0
        for (fn, _), names in zip(self.calls, self.groups):
            if profile:
                self.lib.semicrf_set_profile_events(ctypes_offset(self.handles, 2 * off), 2 * len(names))
            fn()
            off += len(names)
        if profile:
            self.lib.semicrf_set_profile_events(None, 0)
        if self.reduce_fn is not None:
            self.reduce_fn(self.dA, self.dD)

    def time(self, steps, flush):
        t0, t1 = self.torch.cuda.Event(enable_timing=True), self.torch.cuda.Event(enable_timing=True)
        out = []
        for _ in range(steps):
            flush.zero_()                       # L2 flush between timed steps (not timed)
            t0.record(self.stream)
            self.step()
            t1.record(self.stream)
            t1.synchronize()
            out.append(t0.elapsed_time(t1))
        return out

    def kernel_ms(self, steps, flush):
        """Per-kernel times from a separate, untimed pass with events around every launch."""
        kern = {n: 0.0 for n in self.names}
        for _ in range(steps):
            flush.zero_()
            self.step(profile=True)
            self.torch.cuda.synchronize()
            for i, n in enumerate(self.names):
                kern[n] += self.evs[2 * i].elapsed_time(self.evs[2 * i + 1])
        return {n: v / steps for n, v in kern.items()}

    def status(self):
        return self.sc.device_status(self.ws)

    def free(self):
        for k in ("x", "A", "D", "lens", "ws", "S", "nu", "logZ", "dX", "dA", "dD"):
            setattr(self, k, None)


def quick_config(name, dev, flush, peaks, hbm, steps=3, warmup=2):
    """A shorter measurement of the fused step on another named workload."""
    w = wl.make_workload(name, seed=0)
    r = Runner(w, dev, "fused")
    for _ in range(warmup):
        r.step()
    r.torch.cuda.synchronize()
    st = r.status()
    if st != 0:
        raise RuntimeError(f"{name}: device status {r.sc.status_string(st)}")
    ms = statistics.median(r.time(steps, flush))
    rt = roofline_times(w, peaks, hbm)
    sumL, _, _ = algorithmic(w)
    r.free()
    r.torch.cuda.empty_cache()
    return {"B": w.B, "T": w.T, "K": w.K, "C": w.C, "ms_per_step": ms, "value": w.updates / (ms / 1e3),
            "valid_updates_per_s": sumL * w.K * w.C / (ms / 1e3), "steps": steps,
            "frac_sfu": rt["t_sfu_ms"] / ms, "frac_fp64": rt["t_fp64_ms"] / ms, "t_hbm_ms": rt["t_hbm_ms"]}


def run_e2e(args, w, dev, flush, world, reduce_fn):
    """The metric through the public API with host buffers: every step copies the
    inputs in from pinned host memory and every result (log Z, dA, dD, dX) out."""
    import torch
    import torch.distributed as dist
    import semi_markov_crf_prefix_b200 as sc
    B, T, K, C = w.B, w.T, w.K, w.C
    hx = torch.from_numpy(w.x).pin_memory()
    hA = torch.from_numpy(w.A).pin_memory()
    hD = torch.from_numpy(w.D).pin_memory()
    hl = torch.from_numpy(w.lengths).pin_memory()
    h_logZ = torch.empty(B, dtype=torch.float64).pin_memory()
    h_dA = torch.empty((C, C), dtype=torch.float64).pin_memory()
    h_dD = torch.empty((K, C), dtype=torch.float64).pin_memory()
    h_dX = torch.empty((B, T, C), dtype=torch.float32).pin_memory()
    h2d = hx.numel() * 4 + hA.numel() * 4 + hD.numel() * 4 + hl.numel() * 4
    d2h = h_logZ.numel() * 8 + h_dA.numel() * 8 + h_dD.numel() * 8 + h_dX.numel() * 4
    host_entry = world == 1 and args.path == "fused"
    if host_entry:
        stage = sc.new_host_stage(B, T, K, C, device=dev)
        ws = sc.new_workspace(B, T, K, C, sc.WS_TRAIN, device=dev)

        def e2e_step():
            # the C-ABI entry point for host buffers: copies in, scan, forward/backward, copies out
            sc.forward_backward_host(hx, hA, hD, hl, ws, stage, logZ=h_logZ, dA=h_dA, dD=h_dD, dX=h_dX,
                                     want_dX=True)
    else:
        # several ranks (the parameter gradients are summed on the device before the copy out),
        # or the checkpointed pair: device copies around the device step
        run = Runner(w, dev, args.path, args.ckpt, reduce_fn)

        def e2e_step():
            run.x.copy_(hx, non_blocking=True)
            run.A.copy_(hA, non_blocking=True)
            run.D.copy_(hD, non_blocking=True)
            run.lens.copy_(hl, non_blocking=True)
            run.step()
            h_logZ.copy_(run.logZ, non_blocking=True)
            h_dA.copy_(run.dA, non_blocking=True)
            h_dD.copy_(run.dD, non_blocking=True)
            h_dX.copy_(run.dX, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream(dev)
    e_ms = 0.0
    for _ in range(args.steps):
        flush.zero_()
        t0.record(stream)
        e2e_step()
        t1.record(stream)
        t1.synchronize()
        e_ms += t0.elapsed_time(t1)
    if world > 1:
        t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e_ms = float(t.item())
    return {"value": world * w.updates * args.steps / (e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "path": "semicrf_forward_backward_host (x, A, D, lengths in; logZ, dA, dD, dX out)"
            if host_entry else "device copies around the device step"}


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import semi_markov_crf_prefix_b200 as sc
    from semi_markov_crf_prefix_b200.dist import reduce_param_grads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    sc.load_library()

    # unit peaks first, in a process of their own, before this process holds the GPU busy
    peaks_live = live_unit_peaks(local) if (rank == 0 and not args.no_unit_peaks) else None

    w = wl.make_workload(args.config, seed=args.seed, B=args.B, T=args.T)
    if rank > 0:   # data-parallel: every rank its own emissions and lengths, shared A and D
        own = wl.make_workload(args.config, seed=args.seed + 1000 * rank, B=args.B, T=args.T)
        w.x, w.lengths = own.x, own.lengths
    B, T, K, C = w.B, w.T, w.K, w.C
    sumL, terms_pass, bytes_path = algorithmic(w)
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.float32, device=dev)
    reduce_fn = reduce_param_grads if world > 1 else None

    run = Runner(w, dev, args.path, args.ckpt, reduce_fn)
    sc.clear_device_status(run.ws)
    for _ in range(args.warmup):
        run.step()
    torch.cuda.synchronize()
    status = run.status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {sc.status_string(status)}")

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    step_ms = run.time(args.steps, flush)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    total_ms = float(sum(step_ms))
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    clk = clocks.stop() if rank == 0 else None
    kern_ms = run.kernel_ms(args.steps, flush)
    status = run.status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {sc.status_string(status)}")
    launches_per_step = len(run.names)
    ws_bytes = int(run.ws.numel())

    # ---- end to end through the public API with host buffers (inputs in, every result out)
    run.free()                      # the host-buffer step has its own buffers
    torch.cuda.empty_cache()
    e2e = None if args.no_e2e else run_e2e(args, w, dev, flush, world, reduce_fn)
    torch.cuda.empty_cache()

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return None

    # ---- the other path on the same workload, and the other named workloads (rank 0, N = 1)
    peaks_m = measured_peaks() or {}
    hbm = float(peaks_m.get("hbm_gbs", HBM_FALLBACK_GBS))
    hbm_src = "MEASURED_PEAKS.json hbm_gbs" if "hbm_gbs" in peaks_m else "fallback 6650 GB/s"
    sm_max = float((clk or {}).get("sm_max_mhz") or peaks_m.get("sm_max_mhz", SM_MAX_MHZ_FALLBACK))
    unit = peaks_live or derived_unit_peaks(sm_max)
    paths = {args.path: {"ms_per_step": total_ms / args.steps, "kernel_ms_per_step": kern_ms}}
    per_config = {}
    if world == 1 and not args.no_sweep:
        other = "ckpt" if args.path == "fused" else "fused"
        r2 = Runner(w, dev, other, args.ckpt)
        for _ in range(2):
            r2.step()
        torch.cuda.synchronize()
        st = r2.status()
        if st != 0:
            raise RuntimeError(f"{other}: device status {sc.status_string(st)}")
        n2 = max(2, min(args.steps, 5))
        ms2 = statistics.median(r2.time(n2, flush))
        paths[other] = {"ms_per_step": ms2, "value": w.updates / (ms2 / 1e3), "steps": n2,
                        "kernel_ms_per_step": r2.kernel_ms(1, flush)}
        r2.free()
        torch.cuda.empty_cache()
        for name in PER_CONFIG:
            if name == args.config and args.B is None and args.T is None:
                continue
            per_config[name] = quick_config(name, dev, flush, unit, hbm)
    for p in paths.values():
        p["description"] = None
    paths.get("fused", {})["description"] = "semicrf_forward_backward: chains side by side, rows stored"
    if "ckpt" in paths:
        paths["ckpt"]["description"] = (f"semicrf_forward + semicrf_backward: checkpoints every "
                                        f"{args.ckpt or math.ceil(math.sqrt(T))} positions, recompute")

    # ---- roofline of the dominant kernel (the chains): FP64 FMA view, against the measured unit rate
    dom = max(kern_ms, key=kern_ms.get)
    per_launch_ms = kern_ms[dom]
    if dom in ("chains", "fwd_chain", "bwd_chain", "recompute"):
        passes = {"chains": 2, "fwd_chain": 1, "bwd_chain": 1, "recompute": 1}[dom]
        flop = 2 * passes * terms_pass
        achieved = flop / (per_launch_ms / 1e3) / 1e12
        peak = 2 * unit["fp64_fma_per_s"] / 1e12
        roof = {"kernel": dom, "bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "traffic": recorded_traffic(dom, args.config) if args.B is None and args.T is None else None,
                "peak_source": "FP64 FMA, " + unit["source"],
                "work": "2 flop per (log-sum-exp, +) term, sum_b L_b (K*C + C*C) terms per pass "
                        f"({passes} pass(es) in the launch)"}
    else:
        nbytes = 4 * B * T * C + 8 * B * (T + 1) * C
        achieved = nbytes / (per_launch_ms / 1e3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": None, "peak_source": hbm_src}
    ms = total_ms / args.steps
    rt = roofline_times(w, unit, hbm)
    value = world * w.updates * args.steps / (total_ms / 1e3)
    kern_share = {n: round(kern_ms[n] / max(1e-9, sum(kern_ms.values())), 4) for n in run.names}
    edge_bytes = B * T * K * C * C * 4
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.config, "B": B, "T": T, "K": K, "C": C,
                   "path": paths[args.path]["description"], "seed": args.seed,
                   "sum_lengths": sumL, "valid_updates_per_s": world * w.valid_updates * args.steps / (total_ms / 1e3),
                   "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"dp{world}"},
        "roofline": roof,
        "roofline_workload": {**rt, "t_step_ms": ms, "frac_sfu": rt["t_sfu_ms"] / ms, "frac_fp64": rt["t_fp64_ms"] / ms,
                              "primary": "slower of t_hbm (HBM bytes at the copy bandwidth) and t_sfu "
                                         "(one MUFU exp per term at the measured MUFU rate)",
                              "hbm_source": hbm_src},
        "unit_peaks": unit,
        "kernel_ms_per_step": kern_ms,
        "kernel_share": kern_share,
        "paths": paths,
        "memory": {"workspace_bytes": ws_bytes, "edge_tensor_bytes": edge_bytes,
                   "workspace_over_edge_tensor": ws_bytes / edge_bytes},
        "per_config": per_config,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": e2e,
        "clocks": clk,
        "wall_s": wall,
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = oracle_sample(w, budget_s=args.cpu_budget)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return out


# --------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    w = wl.make_workload(args.config, seed=args.seed, B=args.B, T=args.T)
    budget = max(0.5, args.cpu_budget / max(1, args.steps))
    for _ in range(args.warmup if args.warmup < 2 else 1):
        oracle_sample(w, budget_s=0.01)
    vals = []
    info = None
    for _ in range(args.steps):
        info = oracle_sample(w, budget_s=budget)
        vals.append(info["value"])
    value = statistics.median(vals)
    cb = dict(info)
    cb["value"] = value
    cb["sample"] += (f"; each of the {args.steps} steps times one such sample; ms_per_step = one full "
                     f"workload step at the measured rate")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.updates / value * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.config, "B": w.B, "T": w.T, "K": w.K, "C": w.C, "seed": args.seed,
                   "parallelism": "cpu"},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="large", choices=[k for k in wl.CONFIGS if k != "tiny10"])
    ap.add_argument("--path", default="fused", choices=["fused", "ckpt"])
    ap.add_argument("--ckpt", type=int, default=0, help="checkpoint interval (0: ceil(sqrt(T)))")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--B", type=int, default=None, help="override the workload's batch (small profiling cases)")
    ap.add_argument("--T", type=int, default=None, help="override the workload's length (same recipe)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the other path and the other workloads")
    ap.add_argument("--no-unit-peaks", action="store_true", help="derive the unit peaks instead of measuring them")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    out = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
