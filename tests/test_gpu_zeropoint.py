"""Zeropoint (asymmetric) quantization on the GPU against the oracle.

Row quantization is integer work decided by fp32 steps that both sides take
in the same precision, so codes, nd (as fp32 bits), zeropoints and code sums
must match bit for bit. The forward's fp16 output must lie within
2e-3 * max(1, |y|) of the oracle's fp64 value.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_matmul_int8_b200 import _lib
from bit_quantized_matmul_int8_b200 import workloads as wl
from gpu_common import check_y, dev, ensure_built, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def asymmetric_rows(X: np.ndarray) -> np.ndarray:
    """Plant the rows zeropoint quantization exists for, and its degenerate ones."""
    X = X.copy()
    R = X.shape[0]
    f16 = np.float16
    if R > 1:
        X[1] = np.abs(X[1])                               # one-signed (post-ReLU) row
    if R > 2:
        X[2] = (X[2].astype(np.float32) * f16(0.01) + f16(100.0)).astype(f16)  # large offset, small range
    if R > 3:
        X[3] = f16(1.5)                                    # constant row: nd = 1
    if R > 4:
        X[4] = 0                                           # all zero
    if R > 5:
        X[5] = -np.abs(X[5])                               # all non-positive
    if R > 6:
        X[6, :] = f16(-0.25)
        X[6, X.shape[1] // 2] = f16(60.0)                  # one huge value in a constant row
    if R > 7:
        X[7] = (X[7].astype(np.float32) - f16(2000.0)).astype(f16)  # coarse fp16 spacing
    return X


def check_zp_rows(X: np.ndarray, got) -> None:
    Q, ND, ZP, SUM = (host(t) for t in got)
    Qo, NDo, ZPo, SUMo = oracle.zp_quantize_rows(X)
    assert np.array_equal(ND.view(np.uint32), NDo.view(np.uint32)), "nd"
    assert np.array_equal(ZP, ZPo), "zeropoints"
    assert np.array_equal(Q, Qo), "codes"
    assert np.array_equal(SUM, SUMo), "code sums"


ZQCASES = [
    ("tiny", 16, 64),
    ("ragged", 37, 96),
    ("few_long", 5, 12288),          # a CTA per row
    ("wide", 130, 4112),             # a CTA per row, ragged vector count
    ("many_short", 3000, 256),       # a warp per row
    ("many_mid", 1300, 1008),        # a warp per row, K not a multiple of 256
    ("very_long", 9, 65536),
]


@pytest.mark.parametrize("name,R,K", ZQCASES, ids=[c[0] for c in ZQCASES])
def test_zp_quantize_rows_bit_exact(name, R, K):
    w = wl.random_case(71, R, K, 8, n_outliers=3, frac=0.5)
    X = asymmetric_rows(wl.make_x(w))
    check_zp_rows(X, _lib.int8lt_quantize_rows_zp(dev(X)))


@pytest.mark.parametrize("N,K", [(520, 4096), (40, 144), (8, 16)])
def test_zp_prepare_weight_bit_exact(N, K):
    w = wl.random_case(72, 4, K, N)
    W = asymmetric_rows(wl.make_w(w))
    CB, NDB, ZB, SB = _lib.int8lt_prepare_weight_zp(dev(W))
    check_zp_rows(W, (_lib.int8lt_unpack_weight(CB, N, K), NDB, ZB, SB))
    # padding of the blocked layout is zero codes
    assert torch.equal(_lib.int8lt_pack_weight(_lib.int8lt_unpack_weight(CB, N, K)), CB)


def test_zp_codes_span_the_range():
    """Each non-constant row reaches both -127 and 127 (the point of the zeropoint)."""
    w = wl.random_case(73, 64, 1024, 8, n_outliers=2, frac=0.5)
    X = wl.make_x(w)
    X[::2] = np.abs(X[::2])
    Q, _, _, _ = (host(t) for t in _lib.int8lt_quantize_rows_zp(dev(X)))
    assert (Q.min(axis=1) == -127).all() and (Q.max(axis=1) >= 126).all()


def run_zp_forward(w: wl.Workload, rows=None, bias=True):
    X = asymmetric_rows(wl.make_x(w))
    W = wl.make_w(w)
    b = wl.make_bias(w) if bias else None
    CB, NDB, ZB, SB = _lib.int8lt_prepare_weight_zp(dev(W))
    Y = _lib.int8lt_forward_zp(dev(X), CB, NDB, ZB, SB, dev(b) if b is not None else None)
    torch.cuda.synchronize()
    CBo, NDBo, ZBo, SBo = oracle.zp_quantize_rows(W)
    Y64 = oracle.zp_forward(X, CBo, NDBo, ZBo, SBo, b, rows=rows)
    Yg = host(Y)
    if rows is not None:
        Yg = Yg[np.asarray(rows)]
    return Yg, Y64


ZFCASES = [
    wl.random_case(74, 16, 64, 64),                          # decode, one row block
    wl.random_case(75, 1, 1024, 2048),                       # decode, one token
    wl.random_case(76, 7, 3008, 20000),                      # decode, split row blocks
    wl.random_case(77, 17, 256, 40),                         # smallest prefill M
    wl.random_case(78, 300, 512, 264),                       # ragged tiles
    wl.random_case(79, 600, 2048, 1032, has_bias=False),
    wl.random_case(80, 129, 4112, 520),
]


@pytest.mark.parametrize("w", ZFCASES, ids=[w.name for w in ZFCASES])
def test_zp_forward_vs_oracle(w):
    Yg, Y64 = run_zp_forward(w, bias=w.has_bias)
    check_y(Yg, Y64, w.name)


@pytest.fixture
def split_always():
    prev = _lib.int8lt_set_gemm_split(_lib.SPLIT_ALWAYS)
    yield
    _lib.int8lt_set_gemm_split(prev)


def test_zp_forward_split_tiles_vs_oracle(split_always):
    w = wl.random_case(81, 1280, 512, 4096)
    Yg, Y64 = run_zp_forward(w)
    check_y(Yg, Y64, w.name)


def test_zp_forward_sampled_rows_large():
    """A projection-sized call (2048 x 4096 x 4096): sampled rows, all columns."""
    w = wl.random_case(82, 2048, 4096, 4096)
    rows = [0, 1, 2, 3, 4, 5, 6, 7, 255, 256, 1024, 2047]
    Yg, Y64 = run_zp_forward(w, rows=rows)
    check_y(Yg, Y64, w.name)


@pytest.mark.parametrize("M", [5, 300])
def test_zp_halves_equal_forward(M):
    w = wl.random_case(84, M, 512, 264)
    X = dev(asymmetric_rows(wl.make_x(w)))
    b = dev(wl.make_bias(w))
    CB, NDB, ZB, SB = _lib.int8lt_prepare_weight_zp(dev(wl.make_w(w)))
    Y1 = _lib.int8lt_forward_zp(X, CB, NDB, ZB, SB, b)
    ws = _lib.workspace(M, 264, 512, "cuda")
    Y2 = torch.empty_like(Y1)
    _lib.int8lt_forward_zp_quantize(X, 264, ws)
    _lib.int8lt_forward_zp_matmul(M, 512, CB, NDB, ZB, SB, b, Y2, ws)
    assert torch.equal(Y1, Y2)


def test_zp_forward_empty_and_errors():
    Xd = torch.zeros((0, 64), dtype=torch.float16, device="cuda")
    W = dev(wl.make_w(wl.random_case(83, 4, 64, 16)))
    CB, NDB, ZB, SB = _lib.int8lt_prepare_weight_zp(W)
    Y = _lib.int8lt_forward_zp(Xd, CB, NDB, ZB, SB)
    assert Y.shape == (0, 16)
    X = torch.ones((4, 64), dtype=torch.float16, device="cuda")
    ws = _lib.workspace(4, 16, 64, "cuda")
    Y = torch.empty((4, 16), dtype=torch.float16, device="cuda")
    st = _lib.lib().int8lt_forward_zp(X.data_ptr(), 4, 16, 64, CB.data_ptr(), NDB.data_ptr(), None,
                                      SB.data_ptr(), None, Y.data_ptr(), ws.data_ptr(), ws.numel(),
                                      None)
    assert _lib.STATUS[st] == "INT8LT_ERR_NULL"
    st = _lib.lib().int8lt_quantize_rows_zp(X.data_ptr(), 4, 40, None, None, None, None, None)
    assert _lib.STATUS[st] == "INT8LT_ERR_SHAPE"
