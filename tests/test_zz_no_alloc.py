"""The allocation-free prefix scan against the workspace version.

semicrf_prefix_scan_noalloc serves callers that are handed only their input and
output buffers (a plugin or custom-op interface without a workspace hook) or
that must not call cudaMalloc under a fixed memory budget; it keeps its scratch
in a static device array inside the library.  This file is collected last on
purpose, so a failure here comes after every other test has run.  It calls the
entry point twice in a row (the second call reuses the looked-up scratch
address and finds the first call's leftovers in the shared array) and compares
each result with semicrf_prefix_scan.
"""
import ctypes

import numpy as np
import pytest

import semicrf_workloads as wl
from semi_markov_crf_prefix_b200 import _lib

pytestmark = pytest.mark.gpu

ATOL_S = 1e-11   # the tolerance the prefix-scan parity test holds S to


def _run(w):
    import torch
    import semi_markov_crf_prefix_b200 as sc
    dev = torch.device("cuda:0")
    x = torch.from_numpy(w.x).to(dev)
    lens = torch.from_numpy(w.lengths).to(dev)
    S_ref, nu_ref = sc.prefix_scan(x, lens)
    S = torch.full((w.B, w.T + 1, w.C), float("nan"), dtype=torch.float64, device=dev)
    nu = torch.full((w.B, w.C), float("nan"), dtype=torch.float64, device=dev)
    d = _lib.dims(w.B, w.T, 1, w.C)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    st = _lib.load().semicrf_prefix_scan_noalloc(ctypes.byref(d), ctypes.c_void_p(x.data_ptr()),
                                                ctypes.c_void_p(lens.data_ptr()), ctypes.c_void_p(S.data_ptr()),
                                                ctypes.c_void_p(nu.data_ptr()), stream)
    assert st == _lib.SEMICRF_OK, _lib.status_string(st)
    torch.cuda.synchronize()
    return S.cpu().numpy(), nu.cpu().numpy(), S_ref.cpu().numpy(), nu_ref.cpu().numpy()


def test_noalloc_scan_matches_workspace_scan_twice():
    # two different problems back to back through the same static scratch
    for w in (wl.make_workload("ner"), wl.make_workload("large", B=3, T=5000)):
        S, nu, S_ref, nu_ref = _run(w)
        assert np.isfinite(S).all() and np.isfinite(nu).all()
        np.testing.assert_allclose(nu, nu_ref, rtol=0, atol=1e-13)
        np.testing.assert_allclose(S, S_ref, rtol=0, atol=ATOL_S)


def test_noalloc_scan_rejects_oversized_problem():
    d = _lib.dims(1024, 8, 1, 256)      # B*C = 262144 chunk sums > 1 MiB of float64
    p = ctypes.c_void_p(1 << 20)        # never dereferenced: rejected on the host
    st = _lib.load().semicrf_prefix_scan_noalloc(ctypes.byref(d), p, p, p, p, None)
    assert st == _lib.SEMICRF_ERR_UNSUPPORTED_SHAPE
