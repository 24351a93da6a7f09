"""B200-native exact semi-CRF: prefix-sum segment scores, streaming forward-
backward with checkpoints, exact gradients, Viterbi.

Thin binding over ``libsemicrf.so`` (C ABI in ``include/semicrf.h``): this module
only marshals torch CUDA tensors into the library's calls on the current CUDA
stream.  Every step of the computation runs in the library's kernels; there is
no CPU or PyTorch fallback.

Layout (row-major): x float32 [B,T,C]; A float32 [C,C] (from, to); D float32
[K,C] (row d-1); lengths int32 [B]; S float64 [B,T+1,C]; logZ float64 [B];
dX float32 [B,T,C]; dA float64 [C,C]; dD float64 [K,C].
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import (MAX_C, MAX_K, WS_SCAN, WS_TRAIN, WS_VITERBI, SemiCRFError, dims,
                   status_string)

__all__ = ["workspace_bytes", "new_workspace", "new_host_stage", "forward_backward_host", "prefix_scan",
           "prefix_scan_noalloc", "forward", "backward",
           "forward_backward", "viterbi",
           "posteriors", "gold_score", "gold_backward", "nll", "nll_backward", "semicrf_nll",
           "logz_and_grads", "device_status", "clear_device_status", "last_launch_count",
           "SemiCRFError", "status_string", "MAX_C", "MAX_K", "WS_TRAIN", "WS_VITERBI", "WS_SCAN",
           "load_library", "chain_plan"]


def load_library():
    return _lib.load()


def _torch():
    import torch
    return torch


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(device=None):
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, dtype, shape, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need_ws(ws):
    torch = _torch()
    if not isinstance(ws, torch.Tensor) or not ws.is_cuda or ws.dtype != torch.uint8 or not ws.is_contiguous():
        raise TypeError("ws must be a contiguous CUDA uint8 tensor (new_workspace)")


def _same_device(ref, **others):
    """Every tensor given lives on ref's device (None entries are skipped)."""
    for name, t in others.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, expected {ref.device}")


def workspace_bytes(B, T, K, C, what=WS_TRAIN, ckpt_interval=0) -> int:
    d = dims(B, T, K, C, ckpt_interval)
    n = _lib.load().semicrf_workspace_bytes(ctypes.byref(d), int(what))
    if n == 0:
        _lib.check(_lib.load().semicrf_check_dims(ctypes.byref(d)), "workspace_bytes")
    return int(n)


def new_workspace(B, T, K, C, what=WS_TRAIN, ckpt_interval=0, device="cuda"):
    """A device workspace (uint8 tensor, 256-byte aligned by the caching allocator)."""
    torch = _torch()
    n = workspace_bytes(B, T, K, C, what, ckpt_interval)
    return torch.empty(n, dtype=torch.uint8, device=device)


def prefix_scan(x, lengths, ws=None, S=None, nu=None):
    """nu [B,C] and S [B,T+1,C] (float64) from x [B,T,C] float32."""
    torch = _torch()
    B, T, C = x.shape
    _need(x, torch.float32, (B, T, C), "x")
    _need(lengths, torch.int32, (B,), "lengths")
    if ws is None:
        ws = new_workspace(B, T, 1, C, WS_SCAN, device=x.device)
    S = torch.empty((B, T + 1, C), dtype=torch.float64, device=x.device) if S is None else S
    nu = torch.empty((B, C), dtype=torch.float64, device=x.device) if nu is None else nu
    _same_device(x, lengths=lengths, ws=ws, S=S, nu=nu)
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(nu, torch.float64, (B, C), "nu")
    _need_ws(ws)
    d = dims(B, T, 1, C)
    with torch.cuda.device(x.device):
        _lib.check(_lib.load().semicrf_prefix_scan(ctypes.byref(d), _ptr(x), _ptr(lengths), _ptr(S), _ptr(nu),
                                                   _ptr(ws), ws.numel(), _stream(x.device)), "prefix_scan")
    return S, nu


def prefix_scan_noalloc(x, lengths, S=None, nu=None):
    """prefix_scan without a workspace: for callers that cannot allocate device
    scratch.  Uses the library's fixed 1 MiB static scratch (B*C <= 131072);
    concurrent calls on different streams race on it."""
    torch = _torch()
    B, T, C = x.shape
    _need(x, torch.float32, (B, T, C), "x")
    _need(lengths, torch.int32, (B,), "lengths")
    S = torch.empty((B, T + 1, C), dtype=torch.float64, device=x.device) if S is None else S
    nu = torch.empty((B, C), dtype=torch.float64, device=x.device) if nu is None else nu
    _same_device(x, lengths=lengths, S=S, nu=nu)
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(nu, torch.float64, (B, C), "nu")
    d = dims(B, T, 1, C)
    with torch.cuda.device(x.device):
        _lib.check(_lib.load().semicrf_prefix_scan_noalloc(ctypes.byref(d), _ptr(x), _ptr(lengths), _ptr(S),
                                                           _ptr(nu), _stream(x.device)), "prefix_scan_noalloc")
    return S, nu


def forward(S, A, D, lengths, ws=None, ckpt_interval=0, logZ=None):
    """log Z [B] (float64); returns (logZ, ws) -- pass ws unchanged to backward()."""
    torch = _torch()
    B, T1, C = S.shape
    T = T1 - 1
    K = D.shape[0]
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(A, torch.float32, (C, C), "A")
    _need(D, torch.float32, (K, C), "D")
    _need(lengths, torch.int32, (B,), "lengths")
    if ws is None:
        ws = new_workspace(B, T, K, C, WS_TRAIN, ckpt_interval, device=S.device)
    logZ = torch.empty(B, dtype=torch.float64, device=S.device) if logZ is None else logZ
    _need(logZ, torch.float64, (B,), "logZ")
    _need_ws(ws)
    _same_device(S, A=A, D=D, lengths=lengths, logZ=logZ, ws=ws)
    d = dims(B, T, K, C, ckpt_interval)
    with torch.cuda.device(S.device):
        _lib.check(_lib.load().semicrf_forward(ctypes.byref(d), _ptr(S), _ptr(A), _ptr(D), _ptr(lengths),
                                               _ptr(logZ), _ptr(ws), ws.numel(), _stream(S.device)), "forward")
    return logZ, ws


def backward(S, A, D, lengths, ws, grad_logZ=None, ckpt_interval=0, dX=None, dA=None, dD=None):
    """(dX [B,T,C] float32, dA [C,C] float64, dD [K,C] float64) of sum_b g_b logZ_b."""
    torch = _torch()
    B, T1, C = S.shape
    T = T1 - 1
    K = D.shape[0]
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(A, torch.float32, (C, C), "A")
    _need(D, torch.float32, (K, C), "D")
    _need(lengths, torch.int32, (B,), "lengths")
    if grad_logZ is not None:
        _need(grad_logZ, torch.float64, (B,), "grad_logZ")
    dX = torch.empty((B, T, C), dtype=torch.float32, device=S.device) if dX is None else dX
    dA = torch.empty((C, C), dtype=torch.float64, device=S.device) if dA is None else dA
    dD = torch.empty((K, C), dtype=torch.float64, device=S.device) if dD is None else dD
    _need(dX, torch.float32, (B, T, C), "dX")
    _need(dA, torch.float64, (C, C), "dA")
    _need(dD, torch.float64, (K, C), "dD")
    _need_ws(ws)
    _same_device(S, A=A, D=D, lengths=lengths, grad_logZ=grad_logZ, ws=ws, dX=dX, dA=dA, dD=dD)
    d = dims(B, T, K, C, ckpt_interval)
    with torch.cuda.device(S.device):
        _lib.check(_lib.load().semicrf_backward(ctypes.byref(d), _ptr(S), _ptr(A), _ptr(D), _ptr(lengths),
                                                _ptr(grad_logZ), _ptr(ws), ws.numel(), _ptr(dX), _ptr(dA),
                                                _ptr(dD), _stream(S.device)), "backward")
    return dX, dA, dD


def viterbi(S, A, D, lengths, ws=None):
    """(score [B] float64, labels [B,T] int32, seg_start [B,T] uint8)."""
    torch = _torch()
    B, T1, C = S.shape
    T = T1 - 1
    K = D.shape[0]
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(A, torch.float32, (C, C), "A")
    _need(D, torch.float32, (K, C), "D")
    _need(lengths, torch.int32, (B,), "lengths")
    if ws is None:
        ws = new_workspace(B, T, K, C, WS_VITERBI, device=S.device)
    score = torch.empty(B, dtype=torch.float64, device=S.device)
    labels = torch.empty((B, T), dtype=torch.int32, device=S.device)
    seg = torch.empty((B, T), dtype=torch.uint8, device=S.device)
    _need_ws(ws)
    _same_device(S, A=A, D=D, lengths=lengths, ws=ws)
    d = dims(B, T, K, C)
    with torch.cuda.device(S.device):
        _lib.check(_lib.load().semicrf_viterbi(ctypes.byref(d), _ptr(S), _ptr(A), _ptr(D), _ptr(lengths),
                                               _ptr(score), _ptr(labels), _ptr(seg), _ptr(ws), ws.numel(),
                                               _stream(S.device)), "viterbi")
    return score, labels, seg


def forward_backward(S, A, D, lengths, ws=None, grad_logZ=None, logZ=None, dX=None, dA=None, dD=None):
    """(logZ, dX, dA, dD, ws): forward and backward chains side by side, then the
    gradient passes (no checkpoints)."""
    torch = _torch()
    B, T1, C = S.shape
    T = T1 - 1
    K = D.shape[0]
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(A, torch.float32, (C, C), "A")
    _need(D, torch.float32, (K, C), "D")
    _need(lengths, torch.int32, (B,), "lengths")
    if grad_logZ is not None:
        _need(grad_logZ, torch.float64, (B,), "grad_logZ")
    if ws is None:
        ws = new_workspace(B, T, K, C, WS_TRAIN, device=S.device)
    logZ = torch.empty(B, dtype=torch.float64, device=S.device) if logZ is None else logZ
    dX = torch.empty((B, T, C), dtype=torch.float32, device=S.device) if dX is None else dX
    dA = torch.empty((C, C), dtype=torch.float64, device=S.device) if dA is None else dA
    dD = torch.empty((K, C), dtype=torch.float64, device=S.device) if dD is None else dD
    _need(logZ, torch.float64, (B,), "logZ")
    _need(dX, torch.float32, (B, T, C), "dX")
    _need(dA, torch.float64, (C, C), "dA")
    _need(dD, torch.float64, (K, C), "dD")
    _need_ws(ws)
    _same_device(S, A=A, D=D, lengths=lengths, grad_logZ=grad_logZ, ws=ws, logZ=logZ, dX=dX, dA=dA, dD=dD)
    d = dims(B, T, K, C)
    with torch.cuda.device(S.device):
        _lib.check(_lib.load().semicrf_forward_backward(ctypes.byref(d), _ptr(S), _ptr(A), _ptr(D),
                                                        _ptr(lengths), _ptr(grad_logZ), _ptr(ws), ws.numel(),
                                                        _ptr(logZ), _ptr(dX), _ptr(dA), _ptr(dD),
                                                        _stream(S.device)), "forward_backward")
    return logZ, dX, dA, dD, ws


def new_host_stage(B, T, K, C, device="cuda"):
    """Device staging buffer of forward_backward_host (uint8 tensor)."""
    torch = _torch()
    d = dims(B, T, K, C)
    n = int(_lib.load().semicrf_host_stage_bytes(ctypes.byref(d)))
    if n == 0:
        raise ValueError("unsupported dimensions")
    return torch.empty(n, dtype=torch.uint8, device=device)


def forward_backward_host(x, A, D, lengths, ws, stage, grad_logZ=None, logZ=None, dA=None, dD=None, dX=None,
                          want_dX=False):
    """One step from host tensors (pin them for asynchronous copies): the library
    copies x, A, D, lengths (and grad_logZ) to the device, runs prefix_scan and
    forward_backward, and copies logZ, dA, dD (and dX when asked) back, all on the
    current stream of the stage's device.  Returns (logZ, dA, dD, dX or None) as
    host tensors, valid once that stream has synchronised."""
    torch = _torch()
    B, T, C = x.shape
    K = D.shape[0]
    for t, dt, shp, name in ((x, torch.float32, (B, T, C), "x"), (A, torch.float32, (C, C), "A"),
                             (D, torch.float32, (K, C), "D"), (lengths, torch.int32, (B,), "lengths")):
        if t.is_cuda or t.dtype != dt or tuple(t.shape) != shp or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous host {dt} tensor of shape {shp}")
    if grad_logZ is not None and (grad_logZ.is_cuda or grad_logZ.dtype != torch.float64):
        raise TypeError("grad_logZ must be a host float64 tensor")
    pin = torch.cuda.is_available()
    logZ = torch.empty(B, dtype=torch.float64, pin_memory=pin) if logZ is None else logZ
    dA = torch.empty((C, C), dtype=torch.float64, pin_memory=pin) if dA is None else dA
    dD = torch.empty((K, C), dtype=torch.float64, pin_memory=pin) if dD is None else dD
    if want_dX and dX is None:
        dX = torch.empty((B, T, C), dtype=torch.float32, pin_memory=pin)
    for t, dt, shp, name in ((logZ, torch.float64, (B,), "logZ"), (dA, torch.float64, (C, C), "dA"),
                             (dD, torch.float64, (K, C), "dD"), (dX, torch.float32, (B, T, C), "dX"),
                             (grad_logZ, torch.float64, (B,), "grad_logZ")):
        if t is not None and (t.is_cuda or t.dtype != dt or tuple(t.shape) != shp or not t.is_contiguous()):
            raise TypeError(f"{name} must be a contiguous host {dt} tensor of shape {shp}")
    _need_ws(ws)
    _need_ws(stage)
    _same_device(stage, ws=ws)
    d = dims(B, T, K, C)
    with torch.cuda.device(stage.device):
        _lib.check(_lib.load().semicrf_forward_backward_host(
            ctypes.byref(d), _ptr(x), _ptr(A), _ptr(D), _ptr(lengths), _ptr(grad_logZ), _ptr(logZ), _ptr(dX),
            _ptr(dA), _ptr(dD), _ptr(stage), stage.numel(), _ptr(ws), ws.numel(), _stream(stage.device)),
            "forward_backward_host")
    return logZ, dA, dD, dX


def posteriors(S, A, D, lengths, ws, ckpt_interval=0, want_mu=True, want_pstart=True):
    """(mu [B,T,C] float32 or None, pstart [B,T] float32 or None): posterior coverage
    of each label and probability that a segment begins at each position.  ws is
    the workspace of the matching forward()."""
    torch = _torch()
    B, T1, C = S.shape
    T = T1 - 1
    K = D.shape[0]
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(A, torch.float32, (C, C), "A")
    _need(D, torch.float32, (K, C), "D")
    _need(lengths, torch.int32, (B,), "lengths")
    _need_ws(ws)
    _same_device(S, A=A, D=D, lengths=lengths, ws=ws)
    mu = torch.empty((B, T, C), dtype=torch.float32, device=S.device) if want_mu else None
    ps = torch.empty((B, T), dtype=torch.float32, device=S.device) if want_pstart else None
    d = dims(B, T, K, C, ckpt_interval)
    with torch.cuda.device(S.device):
        _lib.check(_lib.load().semicrf_posteriors(ctypes.byref(d), _ptr(S), _ptr(A), _ptr(D), _ptr(lengths),
                                                  _ptr(ws), ws.numel(), _ptr(mu), _ptr(ps), _stream(S.device)),
                   "posteriors")
    return mu, ps


def gold_score(S, A, D, lengths, labels, seg_start, ws):
    """Score [B] float64 of the segmentations given by labels [B,T] int32 and
    seg_start [B,T] uint8 (the Viterbi output format)."""
    torch = _torch()
    B, T1, C = S.shape
    T = T1 - 1
    K = D.shape[0]
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(A, torch.float32, (C, C), "A")
    _need(D, torch.float32, (K, C), "D")
    _need(lengths, torch.int32, (B,), "lengths")
    _need(labels, torch.int32, (B, T), "labels")
    _need(seg_start, torch.uint8, (B, T), "seg_start")
    _need_ws(ws)
    _same_device(S, A=A, D=D, lengths=lengths, labels=labels, seg_start=seg_start, ws=ws)
    score = torch.empty(B, dtype=torch.float64, device=S.device)
    d = dims(B, T, K, C)
    with torch.cuda.device(S.device):
        _lib.check(_lib.load().semicrf_gold_score(ctypes.byref(d), _ptr(S), _ptr(A), _ptr(D), _ptr(lengths),
                                                  _ptr(labels), _ptr(seg_start), _ptr(score), _ptr(ws),
                                                  ws.numel(), _stream(S.device)), "gold_score")
    return score


def gold_backward(lengths, labels, seg_start, ws, dX, dA, dD, grad_score=None):
    """Add the gradient of sum_b g_b score_b of the given segmentations to dX, dA, dD."""
    torch = _torch()
    B, T, C = dX.shape
    K = dD.shape[0]
    _need(dX, torch.float32, (B, T, C), "dX")
    _need(dA, torch.float64, (C, C), "dA")
    _need(dD, torch.float64, (K, C), "dD")
    _need(lengths, torch.int32, (B,), "lengths")
    _need(labels, torch.int32, (B, T), "labels")
    _need(seg_start, torch.uint8, (B, T), "seg_start")
    if grad_score is not None:
        _need(grad_score, torch.float64, (B,), "grad_score")
    _need_ws(ws)
    _same_device(dX, dA=dA, dD=dD, lengths=lengths, labels=labels, seg_start=seg_start, grad_score=grad_score,
                 ws=ws)
    d = dims(B, T, K, C)
    with torch.cuda.device(dX.device):
        _lib.check(_lib.load().semicrf_gold_backward(ctypes.byref(d), _ptr(lengths), _ptr(labels),
                                                     _ptr(seg_start), _ptr(grad_score), _ptr(dX), _ptr(dA),
                                                     _ptr(dD), _ptr(ws), ws.numel(), _stream(dX.device)),
                   "gold_backward")
    return dX, dA, dD


def nll(S, A, D, lengths, labels, seg_start, ws, ckpt_interval=0):
    """(nll, logZ, score) [B] float64: nll = log Z - score of the gold segmentations
    (labels [B,T] int32, seg_start [B,T] uint8), formed on the device; ws keeps the
    forward's checkpoints for nll_backward."""
    torch = _torch()
    B, T1, C = S.shape
    T = T1 - 1
    K = D.shape[0]
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(A, torch.float32, (C, C), "A")
    _need(D, torch.float32, (K, C), "D")
    _need(lengths, torch.int32, (B,), "lengths")
    _need(labels, torch.int32, (B, T), "labels")
    _need(seg_start, torch.uint8, (B, T), "seg_start")
    _need_ws(ws)
    _same_device(S, A=A, D=D, lengths=lengths, labels=labels, seg_start=seg_start, ws=ws)
    out = torch.empty((3, B), dtype=torch.float64, device=S.device)
    d = dims(B, T, K, C, ckpt_interval)
    with torch.cuda.device(S.device):
        _lib.check(_lib.load().semicrf_nll(ctypes.byref(d), _ptr(S), _ptr(A), _ptr(D), _ptr(lengths), _ptr(labels),
                                           _ptr(seg_start), _ptr(out[1]), _ptr(out[2]), _ptr(out[0]), _ptr(ws),
                                           ws.numel(), _stream(S.device)), "nll")
    return out[0], out[1], out[2]


def nll_backward(S, A, D, lengths, labels, seg_start, ws, grad_nll=None, ckpt_interval=0):
    """(dX, dA, dD): gradient of sum_b g_b nll_b (g = grad_nll, None: ones); ws from nll()."""
    torch = _torch()
    B, T1, C = S.shape
    T = T1 - 1
    K = D.shape[0]
    _need(S, torch.float64, (B, T + 1, C), "S")
    _need(A, torch.float32, (C, C), "A")
    _need(D, torch.float32, (K, C), "D")
    _need(lengths, torch.int32, (B,), "lengths")
    _need(labels, torch.int32, (B, T), "labels")
    _need(seg_start, torch.uint8, (B, T), "seg_start")
    if grad_nll is not None:
        _need(grad_nll, torch.float64, (B,), "grad_nll")
    _need_ws(ws)
    _same_device(S, A=A, D=D, lengths=lengths, labels=labels, seg_start=seg_start, ws=ws, grad_nll=grad_nll)
    dX = torch.empty((B, T, C), dtype=torch.float32, device=S.device)
    dA = torch.empty((C, C), dtype=torch.float64, device=S.device)
    dD = torch.empty((K, C), dtype=torch.float64, device=S.device)
    d = dims(B, T, K, C, ckpt_interval)
    with torch.cuda.device(S.device):
        _lib.check(_lib.load().semicrf_nll_backward(ctypes.byref(d), _ptr(S), _ptr(A), _ptr(D), _ptr(lengths),
                                                    _ptr(labels), _ptr(seg_start), _ptr(grad_nll), _ptr(ws),
                                                    ws.numel(), _ptr(dX), _ptr(dA), _ptr(dD), _stream(S.device)),
                   "nll_backward")
    return dX, dA, dD


def semicrf_nll(x, A, D, lengths, labels, seg_start, ckpt_interval=0):
    """Negative log-likelihood log Z_b - score_b(gold) [B] float64, differentiable
    with respect to x, A and D (torch.autograd)."""
    from .training import SemiCRFNLL
    return SemiCRFNLL.apply(x, A, D, lengths, labels, seg_start, ckpt_interval)


def logz_and_grads(x, A, D, lengths, grad_logZ=None, ckpt_interval=0, ws=None):
    """prefix_scan + forward + backward: (logZ, dX, dA, dD, ws)."""
    B, T, C = x.shape
    K = D.shape[0]
    if ws is None:
        ws = new_workspace(B, T, K, C, WS_TRAIN, ckpt_interval, device=x.device)
    S, _ = prefix_scan(x, lengths, ws=ws)
    logZ, ws = forward(S, A, D, lengths, ws=ws, ckpt_interval=ckpt_interval)
    dX, dA, dD = backward(S, A, D, lengths, ws, grad_logZ=grad_logZ, ckpt_interval=ckpt_interval)
    return logZ, dX, dA, dD, ws


def clear_device_status(ws):
    _need_ws(ws)
    with _torch().cuda.device(ws.device):
        _lib.check(_lib.load().semicrf_clear_device_status(_ptr(ws), _stream(ws.device)), "clear_device_status")


def device_status(ws) -> int:
    """Synchronise the current stream and return the workspace's device status code."""
    _need_ws(ws)
    with _torch().cuda.device(ws.device):
        return int(_lib.load().semicrf_get_device_status(_ptr(ws), _stream(ws.device)))


def last_launch_count() -> int:
    return int(_lib.load().semicrf_last_launch_count())


def chain_plan(B, T, K, C, path=0) -> dict:
    """Launch geometry of the chains (semicrf_chain_plan): path 0 the
    forward_backward step, 1 forward, 2 backward."""
    d = dims(B, T, K, C)
    info = (ctypes.c_int32 * 9)()
    _lib.check(_lib.load().semicrf_chain_plan(ctypes.byref(d), int(path), info, 9), "chain_plan")
    keys = ["family", "G", "threads", "labels_per_cta", "lanes_per_label_tr", "lanes_per_label_win",
            "smem_bytes", "resident_clusters", "clusters_needed"]
    return dict(zip(keys, [int(v) for v in info]))
