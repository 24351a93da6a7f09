"""ctypes view of libsemicrf.so (the C ABI declared in include/semicrf.h).

Loading fails loudly when the library has not been built: there is no fallback
path.  Build it with ``python -m semi_markov_crf_prefix_b200.build``.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

LIB_PATH = Path(__file__).resolve().parent / "libsemicrf.so"

SEMICRF_OK = 0
SEMICRF_ERR_INVALID_ARG = 1
SEMICRF_ERR_UNSUPPORTED_SHAPE = 2
SEMICRF_ERR_WORKSPACE_TOO_SMALL = 3
SEMICRF_ERR_CUDA = 4
SEMICRF_ERR_DEVICE_TIMEOUT = 5
SEMICRF_ERR_DEVICE_RANGE = 6
SEMICRF_ERR_INVALID_LENGTH = 7
SEMICRF_ERR_INVALID_SEGMENTATION = 8

WS_TRAIN = 0
WS_VITERBI = 1
WS_SCAN = 2

MAX_C = 256
MAX_K = 4096


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("K", ctypes.c_int32),
                ("C", ctypes.c_int32), ("ckpt_interval", ctypes.c_int32)]


class SemiCRFError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None

# (name, restype, argtypes); P = void*
_P = ctypes.c_void_p
_S = ctypes.c_size_t
_DP = ctypes.POINTER(Dims)
SIGNATURES = {
    "semicrf_workspace_bytes": (ctypes.c_size_t, [_DP, ctypes.c_int32]),
    "semicrf_check_dims": (ctypes.c_int, [_DP]),
    "semicrf_prefix_scan": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _S, _P]),
    "semicrf_prefix_scan_noalloc": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P]),
    "semicrf_forward": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _S, _P]),
    "semicrf_backward": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _S, _P, _P, _P, _P]),
    "semicrf_viterbi": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "semicrf_forward_backward": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _S, _P, _P, _P, _P, _P]),
    "semicrf_host_stage_bytes": (ctypes.c_size_t, [_DP]),
    "semicrf_forward_backward_host": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P, _S, _P]),
    "semicrf_posteriors": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _S, _P, _P, _P]),
    "semicrf_gold_score": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "semicrf_gold_backward": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "semicrf_nll": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "semicrf_nll_backward": (ctypes.c_int, [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P, _P, _P, _P]),
    "semicrf_clear_device_status": (ctypes.c_int, [_P, _P]),
    "semicrf_get_device_status": (ctypes.c_int, [_P, _P]),
    "semicrf_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "semicrf_last_launch_count": (ctypes.c_int32, []),
    "semicrf_chain_plan": (ctypes.c_int, [_DP, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]),
    "semicrf_set_profile_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]),
}


def load():
    """Load libsemicrf.so once; raise if it is missing."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError(f"{LIB_PATH} is not built; run `python -m semi_markov_crf_prefix_b200.build`")
        lib = ctypes.CDLL(str(LIB_PATH))
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().semicrf_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != SEMICRF_OK:
        raise SemiCRFError(status, where)


def dims(B: int, T: int, K: int, C: int, ckpt_interval: int = 0) -> Dims:
    return Dims(int(B), int(T), int(K), int(C), int(ckpt_interval))
