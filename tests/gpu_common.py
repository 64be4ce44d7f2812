"""Shared helpers of the GPU parity tests (CUDA path vs the CPU oracle)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_quantized_matmul_int8_b200 import _lib, build
from bit_quantized_matmul_int8_b200 import workloads as wl

# fp16 output tolerance of the layer: |dY| <= 2e-3 * max(1, |y|), against the
# oracle's fp64 value before its final fp16 rounding.
Y_RTOL = 2e-3


def ensure_built():
    build.build()
    _lib.lib()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def check_y(y_gpu: np.ndarray, y64: np.ndarray, what: str = "") -> None:
    y = y_gpu.astype(np.float64)
    err = np.abs(y - y64)
    tol = Y_RTOL * np.maximum(1.0, np.abs(y64))
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outputs off; worst "
                           f"{float((err / tol).max()):.3f} x tolerance at "
                           f"{np.unravel_index(int(np.argmax(err / tol)), err.shape)}")


def case_inputs(w: wl.Workload, background_threshold=None):
    X = wl.make_x(w, background_threshold=background_threshold)
    W = wl.make_w(w)
    b = wl.make_bias(w)
    return X, W, b


def run_forward(X, W, b, threshold, keep_w=True, rows=None):
    """GPU forward and oracle forward on the same bytes -> (Y_gpu rows, Y64 oracle rows)."""
    Xd, Wd = dev(X), dev(W)
    bd = dev(b) if b is not None else None
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    Y = _lib.int8lt_forward(Xd, CB, SCB, Wd if keep_w else None, threshold, bd)
    torch.cuda.synchronize()
    CBo, SCBo = oracle.prepare_weight(W)
    Y64, _, _ = oracle.forward(X, CBo, SCBo, W if keep_w else None, threshold, b, rows=rows)
    Yg = host(Y)
    if rows is not None:
        Yg = Yg[np.asarray(rows)]
    return Yg, Y64
