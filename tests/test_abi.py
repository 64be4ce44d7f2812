"""The C-ABI library: loads, exports every declared symbol, validates on the host.

CPU only. Every call here fails validation before any CUDA call, so none of
them launches a kernel or dereferences a pointer, with or without a GPU.
"""
import ctypes
import math
import os
import re

import pytest

from bit_quantized_matmul_int8_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "int8lt.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(int8lt_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert names == sorted(_lib.EXPORTS)
    for n in names:
        assert getattr(L, n) is not None


def test_checking_build_exports_every_declared_symbol(L):
    """The checking build (-DINT8LT_DEBUG) is built beside the regular one and
    offers the same C ABI; its extra status code has a name."""
    assert os.path.exists(_lib.CHECK_LIB_PATH)
    C = _lib.lib(_lib.CHECK_LIB_PATH)
    for n in declared_symbols():
        assert getattr(C, n) is not None
    assert C.int8lt_status_string(10).decode().startswith("INT8LT_ERR_BOUNDS")
    assert C.int8lt_version() == L.int8lt_version()


def test_status_strings(L):
    for code, name in _lib.STATUS.items():
        assert L.int8lt_status_string(code).decode().startswith(name)
    assert L.int8lt_version() == 100


def test_workspace_size(L):
    ws = L.int8lt_workspace_size
    assert ws(2048, 4096, 4096) > 2048 * 4096 * 3
    assert ws(16, 49152, 12288) > 16 * 12288
    assert ws(0, 8, 16) > 0                    # empty batch is a valid shape
    for bad in [(1, 8, 8), (1, 8, 24), (1, 12, 16), (-1, 8, 16), (1, 8, 133152)]:
        assert ws(*bad) == 0, bad
    # the prefill layout holds the gathered outlier weights (N x round_up(K, 64) fp16)
    assert ws(17, 4096, 4096) - ws(16, 4096, 4096) > 4096 * 4096 * 2 - 16 * 4096 * 16 * 4


FAKE = 1 << 20   # never dereferenced: each case fails validation first


def fwd(L, X=FAKE, M=32, N=64, K=64, CB=FAKE, SCB=FAKE, Wo=None, thr=6.0, bias=None, Y=FAKE,
        ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = L.int8lt_workspace_size(M, N, K) if M >= 0 else 0
    return L.int8lt_forward(X, M, N, K, CB, SCB, Wo, thr, bias, Y, ws, ws_bytes, None)


def test_forward_validation(L):
    E = _lib.STATUS_CODE
    assert fwd(L, X=None) == E["INT8LT_ERR_NULL"]
    assert fwd(L, Y=None) == E["INT8LT_ERR_NULL"]
    assert fwd(L, ws=None) == E["INT8LT_ERR_NULL"]
    assert fwd(L, K=24) == E["INT8LT_ERR_SHAPE"]
    assert fwd(L, N=12) == E["INT8LT_ERR_SHAPE"]
    assert fwd(L, K=133152) == E["INT8LT_ERR_SHAPE"]
    assert fwd(L, M=-1) == E["INT8LT_ERR_SHAPE"]
    assert fwd(L, X=FAKE + 2) == E["INT8LT_ERR_ALIGN"]
    assert fwd(L, Y=FAKE + 8) == E["INT8LT_ERR_ALIGN"]
    assert fwd(L, Wo=FAKE + 4) == E["INT8LT_ERR_ALIGN"]
    assert fwd(L, bias=FAKE + 1) == E["INT8LT_ERR_ALIGN"]
    assert fwd(L, thr=math.nan) == E["INT8LT_ERR_VALUE"]
    assert fwd(L, thr=-1.0) == E["INT8LT_ERR_VALUE"]
    assert fwd(L, ws_bytes=1024) == E["INT8LT_ERR_WORKSPACE"]


def test_other_entry_validation(L):
    E = _lib.STATUS_CODE
    assert L.int8lt_prepare_weight(None, 8, 16, FAKE, FAKE, None) == E["INT8LT_ERR_NULL"]
    assert L.int8lt_prepare_weight(FAKE, 8, 0, FAKE, FAKE, None) == E["INT8LT_ERR_SHAPE"]
    assert L.int8lt_prepare_weight(FAKE + 2, 8, 16, FAKE, FAKE, None) == E["INT8LT_ERR_ALIGN"]
    ws = L.int8lt_workspace_size(32, 8, 64)
    q = L.int8lt_quantize_rows
    assert q(FAKE, 32, 64, 6.0, FAKE, FAKE, FAKE, None, FAKE, ws, None) == E["INT8LT_ERR_NULL"]
    assert q(FAKE, 32, 60, 6.0, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == E["INT8LT_ERR_SHAPE"]
    assert q(FAKE, 32, 64, math.nan, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == E["INT8LT_ERR_VALUE"]
    assert q(FAKE, 32, 64, 6.0, FAKE, FAKE, FAKE, FAKE, FAKE, 64, None) == E["INT8LT_ERR_WORKSPACE"]
    g = L.int8lt_debug_gemm_i32
    assert g(FAKE, FAKE, 32, 64, 64, None, FAKE, 1 << 30, None) == E["INT8LT_ERR_NULL"]
    assert g(FAKE, FAKE, 32, 64, 40, FAKE, FAKE, 1 << 30, None) == E["INT8LT_ERR_SHAPE"]
    assert L.int8lt_debug_wait_timeout(FAKE, 4096, 10, None) == E["INT8LT_ERR_VALUE"]
    assert L.int8lt_debug_wait_timeout(None, 4096, 10000, None) == E["INT8LT_ERR_NULL"]
    assert L.int8lt_workspace_init(None, 4096, None) == E["INT8LT_ERR_NULL"]
    assert L.int8lt_read_device_status(FAKE, 16, None) == E["INT8LT_ERR_WORKSPACE"]
    bt = L.int8lt_debug_barrier_timeout
    assert bt(None, 1 << 20, 10000, None) == E["INT8LT_ERR_NULL"]
    assert bt(FAKE, 256, 10000, None) == E["INT8LT_ERR_WORKSPACE"]   # header only: no bitmaps
    assert bt(FAKE + 8, 1 << 20, 10000, None) == E["INT8LT_ERR_ALIGN"]
    assert bt(FAKE, 1 << 20, 10, None) == E["INT8LT_ERR_VALUE"]
    assert bt(FAKE, 1 << 20, 2_000_000_000, None) == E["INT8LT_ERR_VALUE"]
    assert L.int8lt_debug_static_scratch_timeout(10, None) == E["INT8LT_ERR_VALUE"]


def _cpu_forward_tensors(M=4, N=64, K=128):
    import torch
    X = torch.zeros((M, K), dtype=torch.float16)
    CB = torch.zeros(_lib.int8lt_weight_bytes(N, K), dtype=torch.int8)
    SCB = torch.zeros(N, dtype=torch.float32)
    W = torch.zeros((N, K), dtype=torch.float16)
    b = torch.zeros(N, dtype=torch.float16)
    Y = torch.zeros((M, N), dtype=torch.float16)
    return X, CB, SCB, W, b, Y


def test_binding_accepts_consistent_forward_arguments(L):
    X, CB, SCB, W, b, Y = _cpu_forward_tensors()
    assert _lib.forward_args(X, CB, SCB, W, b, Y, cuda=False) == (4, 64, 128)
    assert _lib.forward_args(X, CB, SCB, None, None, None, cuda=False) == (4, 64, 128)


@pytest.mark.parametrize("bad", ["Y_short", "Y_wide", "Y_dtype", "Y_strided", "Y_1d", "CB_other_layer",
                                 "W_outlier_shape", "bias_shape", "SCB_dtype", "X_dtype", "X_3d"])
def test_binding_rejects_mismatched_forward_arguments(L, bad):
    """A buffer of the wrong size, type or layout raises in the binding, before
    any call into the library (so before any launch, with or without a GPU)."""
    import torch
    X, CB, SCB, W, b, Y = _cpu_forward_tensors()
    if bad == "Y_short":
        Y = torch.zeros((3, 64), dtype=torch.float16)
    elif bad == "Y_wide":
        Y = torch.zeros((4, 72), dtype=torch.float16)
    elif bad == "Y_dtype":
        Y = torch.zeros((4, 64), dtype=torch.float32)
    elif bad == "Y_strided":
        Y = torch.zeros((64, 4), dtype=torch.float16).t()
    elif bad == "Y_1d":
        Y = torch.zeros(4 * 64, dtype=torch.float16)
    elif bad == "CB_other_layer":
        CB = torch.zeros(_lib.int8lt_weight_bytes(64, 256), dtype=torch.int8)
    elif bad == "W_outlier_shape":
        W = torch.zeros((64, 64), dtype=torch.float16)
    elif bad == "bias_shape":
        b = torch.zeros(32, dtype=torch.float16)
    elif bad == "SCB_dtype":
        SCB = torch.zeros(64, dtype=torch.float16)
    elif bad == "X_dtype":
        X = torch.zeros((4, 128), dtype=torch.float32)
    elif bad == "X_3d":
        X = torch.zeros((1, 4, 128), dtype=torch.float16)
    with pytest.raises(ValueError):
        _lib.forward_args(X, CB, SCB, W, b, Y, cuda=False)


def test_binding_forward_wrappers_validate_first(L, monkeypatch):
    """The forward wrappers run the checks above before they touch the library:
    with the library calls replaced by a recorder, a wrong Y raises and nothing
    is recorded."""
    import torch
    calls = []

    class Recorder:
        def __getattr__(self, name):
            return lambda *a: calls.append(name) or 0

    real = _lib.lib()
    weight_bytes = lambda N, K: int(real.int8lt_weight_bytes(N, K))  # noqa: E731 (host query)
    dev_check = _lib._dev
    monkeypatch.setattr(_lib, "lib", lambda path=None: Recorder())
    monkeypatch.setattr(_lib, "int8lt_weight_bytes", weight_bytes)
    # CPU tensors stand in for device ones: every check but "is it on a GPU" runs
    monkeypatch.setattr(_lib, "_dev", lambda t, dtype, name, shape=None, device=None, cuda=True:
                        dev_check(t, dtype, name, shape, device, False))
    X, CB, SCB, W, b, _ = _cpu_forward_tensors()
    Y = torch.zeros((3, 64), dtype=torch.float16)
    for call in (lambda: _lib.int8lt_forward(X, CB, SCB, W, 6.0, b, Y=Y),
                 lambda: _lib.int8lt_forward_static_scratch(X, CB, SCB, W, Y, 6.0, b),
                 lambda: _lib.int8lt_forward_matmul(4, 128, CB, SCB, W, b, Y, X)):
        with pytest.raises(ValueError, match="Y has shape"):
            call()
    assert calls == []


def test_zeropoint_entry_validation(L):
    E = _lib.STATUS_CODE
    q = L.int8lt_quantize_rows_zp
    assert q(None, 8, 64, FAKE, FAKE, FAKE, FAKE, None) == E["INT8LT_ERR_NULL"]
    assert q(FAKE, 8, 64, FAKE, FAKE, None, FAKE, None) == E["INT8LT_ERR_NULL"]
    assert q(FAKE, 8, 40, FAKE, FAKE, FAKE, FAKE, None) == E["INT8LT_ERR_SHAPE"]
    assert q(FAKE + 8, 8, 64, FAKE, FAKE, FAKE, FAKE, None) == E["INT8LT_ERR_ALIGN"]
    assert q(FAKE, 8, 64, FAKE + 4, FAKE, FAKE, FAKE, None) == E["INT8LT_ERR_ALIGN"]
    assert q(FAKE, 0, 64, None, None, None, None, None) == E["INT8LT_OK"]   # empty: no-op
    p = L.int8lt_prepare_weight_zp
    assert p(FAKE, 12, 64, FAKE, FAKE, FAKE, FAKE, None) == E["INT8LT_ERR_SHAPE"]   # N % 8
    ws = L.int8lt_workspace_size(32, 64, 64)
    f = L.int8lt_forward_zp
    assert f(FAKE, 32, 64, 64, FAKE, FAKE, None, FAKE, None, FAKE, FAKE, ws, None) == E["INT8LT_ERR_NULL"]
    assert f(FAKE, 32, 64, 64, FAKE, FAKE, FAKE + 2, FAKE, None, FAKE, FAKE, ws, None) == E["INT8LT_ERR_ALIGN"]
    assert f(FAKE, 32, 64, 40, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, ws, None) == E["INT8LT_ERR_SHAPE"]
    assert f(FAKE, 32, 64, 64, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 64, None) == E["INT8LT_ERR_WORKSPACE"]
    assert f(FAKE, 0, 64, 64, None, None, None, None, None, None, None, 0, None) == E["INT8LT_OK"]
    h = L.int8lt_forward_zp_quantize
    assert h(None, 32, 64, 64, FAKE, ws, None) == E["INT8LT_ERR_NULL"]
    assert h(FAKE, 32, 64, 64, FAKE, 64, None) == E["INT8LT_ERR_WORKSPACE"]
    m = L.int8lt_forward_zp_matmul
    assert m(32, 64, 64, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, ws, None) == E["INT8LT_ERR_NULL"]
    assert m(32, 64, 64, FAKE, FAKE, FAKE, FAKE, None, FAKE + 8, FAKE, ws, None) == E["INT8LT_ERR_ALIGN"]


def test_layer_memory_accounting(L):
    # "LLM.int8() paper summary", "Int8 Matrix Multiplication at Scale": about
    # half the memory of the fp16 layer once the fp16 weight is dropped.
    for N, K in [(4096, 4096), (16384, 4096), (4096, 16384), (49152, 12288), (36864, 12288)]:
        fp16 = 2 * N * K
        b = L.int8lt_layer_bytes(N, K, 0)
        assert b == L.int8lt_weight_bytes(N, K) + 4 * N == N * K + 4 * N
        assert 0.5 <= b / fp16 <= 0.5 + 1e-3
        assert L.int8lt_layer_bytes(N, K, 1) == b + fp16
    # the blocked layout pads to 32 channels x 128 bytes
    assert L.int8lt_weight_bytes(40, 136) == 2 * 2 * 4096
    assert L.int8lt_layer_bytes(40, 136, 0) == 2 * 2 * 4096 + 160
    assert L.int8lt_weight_bytes(-1, 16) == 0 and L.int8lt_weight_bytes(8, 0) == 0
    assert L.int8lt_layer_bytes(-1, 16, 0) == 0 and L.int8lt_layer_bytes(8, 0, 1) == 0


def test_weight_layout_entry_validation(L):
    E = _lib.STATUS_CODE
    assert L.int8lt_weight_bytes(1, 1) == 4096 and L.int8lt_weight_bytes(33, 129) == 4 * 4096
    assert L.int8lt_weight_bytes(0, 16) == 0
    p, u = L.int8lt_pack_weight, L.int8lt_unpack_weight
    assert p(None, 8, 16, FAKE, None) == E["INT8LT_ERR_NULL"]
    assert p(FAKE, 8, 16, None, None) == E["INT8LT_ERR_NULL"]
    assert p(FAKE, 8, 0, FAKE, None) == E["INT8LT_ERR_SHAPE"]
    assert p(FAKE, -1, 16, FAKE, None) == E["INT8LT_ERR_SHAPE"]
    assert p(FAKE, 8, 16, FAKE + 8, None) == E["INT8LT_ERR_ALIGN"]      # blocked codes: 16 bytes
    assert p(FAKE + 8, 8, 16, FAKE, None) == E["INT8LT_ERR_ALIGN"]      # rows, K % 16 == 0: 16 bytes
    assert u(FAKE + 8, 8, 16, FAKE, None) == E["INT8LT_ERR_ALIGN"]
    assert p(None, 0, 16, None, None) == E["INT8LT_OK"]                 # empty: no-op


def test_product_path_does_not_touch_oracle():
    pkg = os.path.join(ROOT, "bit_quantized_matmul_int8_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "liboracle" not in src and "int8lt_oracle" not in src, f
