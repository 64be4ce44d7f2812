"""The allocation-free decode entry point against the regular forward.

int8lt_forward_static_scratch exists for callers that cannot give the layer a
workspace (a plugin handed only its input and output buffers, a runtime whose
device memory belongs to its own pool, a decode loop that must not call
cudaMalloc because it can synchronize the device). It must produce what
int8lt_forward produces, call after call, although every call reuses the same
fixed device array. This file is collected last so that a run stopping at the
first failure has already run every other test; it also passes on its own in
a fresh process (the array is set up by the first call on the device).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_matmul_int8_b200 import _lib
from bit_quantized_matmul_int8_b200 import workloads as wl
from gpu_common import case_inputs, check_y, dev, ensure_built, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _layer(w, keep_w=True):
    X, W, b = case_inputs(w)
    Wd = dev(W)
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    return X, W, (Wd if keep_w else None), CB, SCB, b


@pytest.mark.parametrize("M,K,N,keep_w", [(1, 1024, 2048, True), (4, 768, 312, False),
                                          (16, 4096, 1024, True), (16, 1024, 40000, True)])
def test_matches_forward_on_two_calls_in_a_row(M, K, N, keep_w):
    w = wl.random_case(90 + M, M, K, N, n_outliers=4, frac=1.0)
    X, W, Wo, CB, SCB, b = _layer(w, keep_w)
    bd = dev(b) if b is not None else None
    CBo, SCBo = oracle.prepare_weight(W)
    # a second input with a different outlier set, so the second call must not
    # reuse anything the first call left in the shared array
    X2 = X.copy()
    X2[:, 5] = 30.0
    for x in (X, X2):
        xd = dev(x)
        ref = _lib.int8lt_forward(xd, CB, SCB, Wo, 6.0, bd)
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        _lib.int8lt_forward_static_scratch(xd, CB, SCB, Wo, Y, 6.0, bd)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: the same bits
        assert torch.equal(Y, ref), "static scratch differs from int8lt_forward"
        Y64, _, _ = oracle.forward(x, CBo, SCBo, W if keep_w else None, 6.0, b)
        check_y(host(Y), Y64, "static scratch vs the oracle")
    assert _lib.int8lt_static_scratch_read_status() == 0


def test_status_reports_a_timeout_and_restores_the_array():
    """A wait that runs out on the device is reported by the status call, which
    also puts the array's header back in order: the next call is correct. The
    shape (16 tokens, 8192 channels) is one whose quantize pass spreads over
    many blocks and meets at the grid barrier whose counts the timeout upsets."""
    M, K, N = 16, 4096, 8192
    w = wl.random_case(97, M, K, N, n_outliers=3, frac=1.0)
    X, W, Wo, CB, SCB, b = _layer(w)
    bd = dev(b)
    xd = dev(X)
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    _lib.int8lt_forward_static_scratch(xd, CB, SCB, Wo, Y, 6.0, bd)   # the array is set up
    assert _lib.int8lt_static_scratch_read_status() == 0
    _lib.int8lt_debug_static_scratch_timeout(1_000_000)               # 1 ms, cannot complete
    assert _lib.int8lt_static_scratch_read_status() == _lib.STATUS_CODE["INT8LT_ERR_TIMEOUT"]
    assert _lib.int8lt_static_scratch_read_status() == 0             # the read cleared it
    ref = _lib.int8lt_forward(xd, CB, SCB, Wo, 6.0, bd)
    for _ in range(2):
        Y.fill_(float("nan"))
        _lib.int8lt_forward_static_scratch(xd, CB, SCB, Wo, Y, 6.0, bd)
        torch.cuda.synchronize()
        assert torch.equal(Y, ref)
    assert _lib.int8lt_static_scratch_read_status() == 0


def test_rejects_calls_beyond_the_array():
    L = _lib.lib()
    E = _lib.STATUS_CODE["INT8LT_ERR_TOO_LARGE"]
    fake = 1 << 20   # never dereferenced: rejected before any launch
    assert L.int8lt_forward_static_scratch(fake, 17, 64, 64, fake, fake, None, 6.0, None, fake,
                                           None) == E
    assert L.int8lt_forward_static_scratch(fake, 16, 200000, 16384, fake, fake, None, 6.0, None,
                                           fake, None) == E
    assert _lib.int8lt_workspace_size(16, 200000, 16384) > (8 << 20)
