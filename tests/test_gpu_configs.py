"""Parity at the full sizes of every benchmark configuration.

The CUDA path runs exactly as bench.py runs it (int8lt_forward on the whole
workload, fp16 weight kept for the outlier columns). Every expected value
comes from the oracle fed with the workload's own inputs (X, W, bias) and its
own weight codes; no array a CUDA entry produced is ever passed to the
oracle. The oracle cannot recompute a full 8192 x 12288 x 36864 product in
test time, so it checks:
  * the outlier set, CA and SCA over the whole X (bit-exact), and that the
    outlier set is the planted one;
  * CB (unpacked from the blocked layout) and SCB over the whole W
    (bit-exact);
  * the int32 accumulators C = CA CB^T on sampled rows, one per 256-row tile
    of the prefill GEMM (bit-exact), through the same kernels as the forward;
  * Y on the same rows, every output channel, against the oracle's fp64
    forward of those rows (fp16 tolerance).
"""
import functools
import math

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_matmul_int8_b200 import _lib
from bit_quantized_matmul_int8_b200 import workloads as wl
from gpu_common import check_y, dev, ensure_built, host

CONFIGS = [n for n in wl.WORKLOADS if n != "tiny_16x64x64"]
TILE_M = 256     # rows of one prefill GEMM output tile


@pytest.fixture(scope="module")
def _built():
    ensure_built()


@functools.lru_cache(maxsize=1)
def _layer(wid: int, N: int, K: int, sigma: float):
    """The workload's weight and the oracle's codes for it (shared by the QKV sweep)."""
    w = wl.Workload("w", 1, K, N, 0, 0.0, sigma_w=sigma, wid=wid)
    W = wl.make_w(w)
    CBo, SCBo = oracle.prepare_weight(W)
    return W, CBo, SCBo


_X_CACHE: dict = {}


def _acts(w: wl.Workload) -> np.ndarray:
    """X of a workload; the threshold = +inf variants reuse the thresholded data."""
    key = (w.M, w.K, w.N, w.n_outliers, w.outlier_frac, w.outlier_lo, w.outlier_hi, w.seed, w.wid)
    if key not in _X_CACHE:
        _X_CACHE.clear()
        _X_CACHE[key] = wl.make_x(w)
    return _X_CACHE[key]


def sample_rows(M: int, seed: int, cap: int = 32) -> np.ndarray:
    """One row from each 256-row tile of the output (a random offset inside it),
    the first and last row included; every row when M <= 16."""
    if M <= 16:
        return np.arange(M, dtype=np.int64)
    rng = np.random.default_rng(seed)
    tiles = math.ceil(M / TILE_M)
    pick = np.linspace(0, tiles - 1, min(tiles, cap)).round().astype(np.int64)
    rows = {0, M - 1}
    for t in pick:
        lo, hi = int(t) * TILE_M, min(M, (int(t) + 1) * TILE_M)
        rows.add(int(rng.integers(lo, hi)))
    return np.array(sorted(rows), dtype=np.int64)


def test_sample_rows_cover_every_tile():
    for M in (2048, 4096, 8192):
        r = sample_rows(M, 0)
        assert len(set((r // TILE_M).tolist())) == min(M // TILE_M, 32)
        assert r[0] == 0 and r[-1] == M - 1
    assert sample_rows(16, 0).tolist() == list(range(16))


@pytest.mark.gpu
@pytest.mark.parametrize("name", CONFIGS)
def test_full_size_config(name, _built):
    w = wl.WORKLOADS[name]
    X = _acts(w)
    W, CBo, SCBo = _layer(w.wid, w.N, w.K, w.sigma_w)
    b = wl.make_bias(w)
    Xd, Wd = dev(X), dev(W)
    bd = dev(b) if b is not None else None
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    ws = _lib.workspace(w.M, w.N, w.K)
    Y = _lib.int8lt_forward(Xd, CB, SCB, Wd, w.threshold, bd, ws=ws)
    torch.cuda.synchronize()
    assert _lib.int8lt_read_device_status(ws) == 0

    # CB / SCB over the whole weight
    CBrows = _lib.int8lt_unpack_weight(CB, w.N, w.K)
    assert np.array_equal(host(CBrows), CBo)
    del CBrows
    assert np.array_equal(host(SCB).view(np.uint32), SCBo.view(np.uint32))

    # outlier set, CA, SCA over the whole X
    CA, SCA, idx = _lib.int8lt_quantize_rows(Xd, w.threshold)
    CAo, SCAo, idxo = oracle.quantize_rows(X, w.threshold)
    want = wl.outlier_columns(w) if math.isfinite(w.threshold) else np.zeros(0, np.int64)
    assert idxo.tolist() == want.tolist()
    assert np.array_equal(host(idx), idxo)
    assert np.array_equal(host(SCA).view(np.uint32), SCAo.view(np.uint32))
    assert np.array_equal(host(CA), CAo)

    # int32 accumulators on sampled rows (same kernel as the forward's matmul)
    rows = sample_rows(w.M, 2)
    C = _lib.int8lt_debug_gemm_i32(CA, CB, w.N, ws=ws)
    Cs = host(C[torch.from_numpy(rows).cuda()])
    del C
    assert np.array_equal(Cs, oracle.gemm_i32(CAo[rows], CBo))

    # Y on the sampled rows, every output channel
    Y64, _, n = oracle.forward(X, CBo, SCBo, W, w.threshold, b, rows=rows)
    assert n == len(want)
    check_y(host(Y)[rows], Y64, name)
