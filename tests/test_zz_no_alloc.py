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
    return X, (Wd if keep_w else None), CB, SCB, (dev(b) if b is not None else None)


@pytest.mark.parametrize("M,K,N,keep_w", [(1, 1024, 2048, True), (4, 768, 312, False),
                                          (16, 4096, 1024, True), (16, 1024, 40000, True)])
def test_matches_forward_on_two_calls_in_a_row(M, K, N, keep_w):
    w = wl.random_case(90 + M, M, K, N, n_outliers=4, frac=1.0)
    X, Wo, CB, SCB, b = _layer(w, keep_w)
    # a second input with a different outlier set, so the second call must not
    # reuse anything the first call left in the shared array
    X2 = X.copy()
    X2[:, 5] = 30.0
    for x in (X, X2):
        xd = dev(x)
        ref = _lib.int8lt_forward(xd, CB, SCB, Wo, 6.0, b)
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        _lib.int8lt_forward_static_scratch(xd, CB, SCB, Wo, Y, 6.0, b)
        torch.cuda.synchronize()
        check_y(host(Y), host(ref).astype(np.float64), "static scratch vs int8lt_forward")


def test_rejects_calls_beyond_the_array():
    L = _lib.lib()
    E = _lib.STATUS_CODE["INT8LT_ERR_TOO_LARGE"]
    fake = 1 << 20   # never dereferenced: rejected before any launch
    assert L.int8lt_forward_static_scratch(fake, 17, 64, 64, fake, fake, None, 6.0, None, fake,
                                           None) == E
    assert L.int8lt_forward_static_scratch(fake, 16, 200000, 16384, fake, fake, None, 6.0, None,
                                           fake, None) == E
    assert _lib.int8lt_workspace_size(16, 200000, 16384) > (8 << 20)
