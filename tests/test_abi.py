"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, sizes workspaces, and rejects bad arguments on the host before any
launch (no compute call is made here)."""
import ctypes
import re
from pathlib import Path

import pytest

from semi_markov_crf_prefix_b200 import _lib
from semi_markov_crf_prefix_b200 import build as build_mod

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return _lib.load()


def declared_functions():
    text = (ROOT / "include" / "semicrf.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(semicrf_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_status_strings(lib):
    for code in range(8):
        s = _lib.status_string(code)
        assert s and s != "unknown status"
    assert _lib.status_string(99) == "unknown status"


def _d(B, T, K, C, ck=0):
    return ctypes.byref(_lib.dims(B, T, K, C, ck))


def test_check_dims(lib):
    assert lib.semicrf_check_dims(_d(2, 64, 8, 4)) == _lib.SEMICRF_OK
    assert lib.semicrf_check_dims(None) == _lib.SEMICRF_ERR_INVALID_ARG
    for bad in [(0, 64, 8, 4), (2, 0, 8, 4), (2, 64, 0, 4), (2, 64, 8, 0), (2, 64, 8, 4, -1)]:
        assert lib.semicrf_check_dims(_d(*bad)) == _lib.SEMICRF_ERR_INVALID_ARG, bad
    assert lib.semicrf_check_dims(_d(2, 64, 8, _lib.MAX_C + 1)) == _lib.SEMICRF_ERR_UNSUPPORTED_SHAPE
    assert lib.semicrf_check_dims(_d(2, 64, _lib.MAX_K + 1, 4)) == _lib.SEMICRF_ERR_UNSUPPORTED_SHAPE
    # every named workload shape is supported
    for shape in [(2, 64, 8, 4), (32, 512, 16, 17), (16, 4000, 64, 128), (1, 100000, 1000, 24),
                  (4, 200000, 512, 256), (1, 1000000, 200, 24)]:
        assert lib.semicrf_check_dims(_d(*shape)) == _lib.SEMICRF_OK, shape


def test_workspace_bytes(lib):
    tr = lib.semicrf_workspace_bytes(_d(2, 64, 8, 4), _lib.WS_TRAIN)
    vi = lib.semicrf_workspace_bytes(_d(2, 64, 8, 4), _lib.WS_VITERBI)
    sc = lib.semicrf_workspace_bytes(_d(2, 64, 8, 4), _lib.WS_SCAN)
    assert 0 < sc < vi < tr
    assert tr % 256 == 0
    assert lib.semicrf_workspace_bytes(_d(0, 64, 8, 4), _lib.WS_TRAIN) == 0
    assert lib.semicrf_workspace_bytes(_d(2, 64, 8, 4), 7) == 0
    # more checkpoints (smaller interval) never shrink the workspace
    a = lib.semicrf_workspace_bytes(_d(2, 4096, 16, 17, 1), _lib.WS_TRAIN)
    b = lib.semicrf_workspace_bytes(_d(2, 4096, 16, 17, 64), _lib.WS_TRAIN)
    assert a > b
    # the largest named workload fits comfortably in one B200's HBM
    big = lib.semicrf_workspace_bytes(_d(4, 200000, 512, 256), _lib.WS_TRAIN)
    assert 0 < big < 16 * 2**30


def test_host_validation_before_launch(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)          # never dereferenced: every call below fails validation first
    d = _d(2, 64, 8, 4)
    tr = lib.semicrf_workspace_bytes(d, _lib.WS_TRAIN)
    # workspace too small
    assert lib.semicrf_forward(d, fake, fake, fake, fake, fake, fake, 16, None) == \
        _lib.SEMICRF_ERR_WORKSPACE_TOO_SMALL
    assert lib.semicrf_backward(d, fake, fake, fake, fake, None, fake, tr - 1, fake, fake, fake, None) == \
        _lib.SEMICRF_ERR_WORKSPACE_TOO_SMALL
    # null workspace / misaligned workspace / null data pointers
    assert lib.semicrf_forward(d, fake, fake, fake, fake, fake, None, tr, None) == _lib.SEMICRF_ERR_INVALID_ARG
    assert lib.semicrf_forward(d, fake, fake, fake, fake, fake, P((1 << 20) + 8), tr, None) == \
        _lib.SEMICRF_ERR_INVALID_ARG
    assert lib.semicrf_forward(d, None, fake, fake, fake, fake, fake, tr, None) == _lib.SEMICRF_ERR_INVALID_ARG
    assert lib.semicrf_backward(d, fake, fake, fake, fake, None, fake, tr, None, fake, fake, None) == \
        _lib.SEMICRF_ERR_INVALID_ARG
    assert lib.semicrf_prefix_scan(d, None, fake, fake, fake, fake, tr, None) == _lib.SEMICRF_ERR_INVALID_ARG
    vi = lib.semicrf_workspace_bytes(d, _lib.WS_VITERBI)
    assert lib.semicrf_viterbi(d, fake, fake, fake, fake, fake, fake, None, fake, vi, None) == \
        _lib.SEMICRF_ERR_INVALID_ARG
    # bad dims
    assert lib.semicrf_forward(_d(2, 64, 8, 300), fake, fake, fake, fake, fake, fake, tr, None) == \
        _lib.SEMICRF_ERR_UNSUPPORTED_SHAPE
    # host-buffer step: stage sizing, short / null / misaligned stage, null host pointers
    hs = lib.semicrf_host_stage_bytes(d)
    assert hs > 0 and hs % 256 == 0 and lib.semicrf_host_stage_bytes(_d(0, 64, 8, 4)) == 0
    fbh = lib.semicrf_forward_backward_host
    assert fbh(d, fake, fake, fake, fake, None, fake, None, fake, fake, fake, hs - 1, fake, tr, None) == \
        _lib.SEMICRF_ERR_WORKSPACE_TOO_SMALL
    assert fbh(d, fake, fake, fake, fake, None, fake, None, fake, fake, None, hs, fake, tr, None) == \
        _lib.SEMICRF_ERR_INVALID_ARG
    assert fbh(d, fake, fake, fake, fake, None, fake, None, fake, fake, P((1 << 20) + 8), hs, fake, tr, None) == \
        _lib.SEMICRF_ERR_INVALID_ARG
    assert fbh(d, None, fake, fake, fake, None, fake, None, fake, fake, fake, hs, fake, tr, None) == \
        _lib.SEMICRF_ERR_INVALID_ARG
    assert lib.semicrf_get_device_status(None, None) == _lib.SEMICRF_ERR_INVALID_ARG
    assert lib.semicrf_clear_device_status(None, None) == _lib.SEMICRF_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    import semi_markov_crf_prefix_b200 as sc
    x = torch.zeros(1, 4, 2)
    with pytest.raises(TypeError):
        sc.prefix_scan(x, torch.ones(1, dtype=torch.int32))
