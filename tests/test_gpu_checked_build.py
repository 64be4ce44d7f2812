"""The checking build (libint8lt_check.so, compiled with -DINT8LT_DEBUG).

Its kernels check the index of their computed global accesses (outlier ranks
into Xo and the outlier list, outlier columns into the fp16 weight, the decode
GEMV's partial sums, counters and outputs, the raw int32 stores) and record a
failed check as INT8LT_ERR_BOUNDS in the device status, skipping the access.
On valid inputs no check may fail, and the results must be the regular
build's, bit for bit: the checks change no arithmetic.
"""
import pytest
import torch

from bit_quantized_matmul_int8_b200 import _lib
from bit_quantized_matmul_int8_b200 import workloads as wl
from gpu_common import case_inputs, dev, ensure_built

pytestmark = pytest.mark.gpu

CASES = [
    wl.random_case(201, 1, 4096, 2048, n_outliers=5, frac=1.0),      # decode, cluster pass
    wl.random_case(202, 16, 2064, 9992, n_outliers=7, frac=1.0),     # decode, cooperative pass
    wl.random_case(203, 300, 1040, 520, n_outliers=9, frac=0.4),     # prefill, ragged tiles
    wl.random_case(204, 610, 10256, 264, n_outliers=5, frac=0.4),    # prefill, long rows
    wl.random_case(205, 77, 4096, 1032, n_outliers=40, frac=0.5),    # two outlier k-blocks
]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _run(c, keep_w):
    X, W, b = case_inputs(c)
    Xd, Wd, bd = dev(X), dev(W), dev(b)
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    ws = _lib.workspace(c.M, c.N, c.K)
    Y = _lib.int8lt_forward(Xd, CB, SCB, Wd if keep_w else None, 6.0, bd, ws=ws)
    CA, SCA, idx = _lib.int8lt_quantize_rows(Xd, 6.0)
    C32 = _lib.int8lt_debug_gemm_i32(CA, CB, c.N)
    CBz, NDB, ZB, SB = _lib.int8lt_prepare_weight_zp(Wd)
    Yz = _lib.int8lt_forward_zp(Xd, CBz, NDB, ZB, SB, bd, ws=ws)
    torch.cuda.synchronize()
    status = _lib.int8lt_read_device_status(ws)
    return [Y, CA, SCA, idx, C32, Yz], status


@pytest.mark.parametrize("keep_w", [True, False])
@pytest.mark.parametrize("c", CASES, ids=[c.name for c in CASES])
def test_checking_build_matches_and_reports_nothing(c, keep_w):
    ref, st = _run(c, keep_w)
    assert st == 0
    with _lib.using_library(_lib.CHECK_LIB_PATH):
        got, st_chk = _run(c, keep_w)
    assert st_chk == 0, _lib.STATUS.get(st_chk)
    for r, g in zip(ref, got):
        assert torch.equal(r, g)
