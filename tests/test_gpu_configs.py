"""Parity at the full sizes of every benchmark configuration, on sampled outputs.

The CUDA path runs exactly as bench.py runs it (int8lt_forward on the whole
workload). The oracle cannot recompute a full 8192 x 12288 x 36864 product in
test time, so it checks:
  * the outlier set, CA and SCA over the whole X (bit-exact);
  * CB/SCB on sampled weight rows (bit-exact);
  * the int32 accumulators on sampled rows of C = CA CB^T (bit-exact);
  * Y on sampled rows against the oracle forward of those rows (fp16 tolerance),
and, at every size, that the outlier set is the planted one.
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

pytestmark = pytest.mark.gpu

CONFIGS = [n for n in wl.WORKLOADS if n != "tiny_16x64x64"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


@functools.lru_cache(maxsize=2)
def _weights(wid: int, N: int, K: int, sigma: float):
    w = wl.Workload("w", 1, K, N, 0, 0.0, sigma_w=sigma, wid=wid)
    return wl.make_w(w)


_X_CACHE: dict = {}


def _acts(w: wl.Workload) -> np.ndarray:
    """X of a workload; the threshold = +inf variants reuse the thresholded data."""
    key = (w.M, w.K, w.N, w.n_outliers, w.outlier_frac, w.outlier_lo, w.outlier_hi, w.seed, w.wid)
    if key not in _X_CACHE:
        _X_CACHE.clear()
        _X_CACHE[key] = wl.make_x(w)
    return _X_CACHE[key]


def _sample_rows(M: int, k: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = {0, M - 1}
    rows.update(rng.integers(0, M, size=k).tolist())
    return np.array(sorted(rows)[: k + 2], dtype=np.int64)


@pytest.mark.parametrize("name", CONFIGS)
def test_full_size_config(name):
    w = wl.WORKLOADS[name]
    X = _acts(w)
    W = _weights(w.wid, w.N, w.K, w.sigma_w)
    b = wl.make_bias(w)
    Xd, Wd = dev(X), dev(W)
    bd = dev(b) if b is not None else None
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    ws = _lib.workspace(w.M, w.N, w.K)
    Y = _lib.int8lt_forward(Xd, CB, SCB, Wd, w.threshold, bd, ws=ws)
    torch.cuda.synchronize()
    assert _lib.int8lt_read_device_status(ws) == 0

    # outlier set, CA, SCA over the whole X
    CA, SCA, idx = _lib.int8lt_quantize_rows(Xd, w.threshold)
    CAo, SCAo, idxo = oracle.quantize_rows(X, w.threshold)
    assert np.array_equal(host(idx), idxo)
    want = wl.outlier_columns(w) if math.isfinite(w.threshold) else np.zeros(0, np.int64)
    assert host(idx).tolist() == want.tolist()
    assert np.array_equal(host(SCA), SCAo)
    assert np.array_equal(host(CA), CAo)

    # CB / SCB on sampled weight rows
    CBrows = _lib.int8lt_unpack_weight(CB, w.N, w.K)
    jr = _sample_rows(w.N, 64, 1)
    CBo, SCBo = oracle.prepare_weight(W[jr])
    assert np.array_equal(host(CBrows[torch.from_numpy(jr).cuda()]), CBo)
    assert np.array_equal(host(SCB[torch.from_numpy(jr).cuda()]), SCBo)

    # int32 accumulators on sampled rows (same kernel as the forward's matmul)
    rows = _sample_rows(w.M, 3 if w.M * w.N * w.K > 1e12 else 6, 2)
    C = _lib.int8lt_debug_gemm_i32(CA, CB, w.N, ws=ws)
    Cs = host(C[torch.from_numpy(rows).cuda()])
    del C
    CBfull = host(CBrows)
    del CBrows
    Cref = oracle.gemm_i32(CAo[rows], CBfull)
    assert np.array_equal(Cs, Cref)

    # Y on sampled rows against the oracle forward of those rows
    CBo_full, SCBo_full = CBfull, host(SCB)
    Y64, _, n = oracle.forward(X, CBo_full, SCBo_full, W, w.threshold, b, rows=rows)
    assert n == len(want)
    check_y(host(Y)[rows], Y64, name)
