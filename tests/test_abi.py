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
