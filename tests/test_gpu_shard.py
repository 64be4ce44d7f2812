"""Output-channel sharding on one GPU: each rank's forward, stitched, is the layer's.

A layer split by output channel (bit_quantized_matmul_int8_b200.shard) gives
rank r the rows [n0, n1) of W -- its slice of the prepared codes CB (whole row
blocks of the blocked weight layout), of SCB, of the fp16 weight and of the
bias -- and the whole of X. The outlier set depends on X alone, so each shard's
int8lt_forward must produce exactly the layer's columns [n0, n1): the stitched
Y is bit-identical to the unsharded forward and within the fp16 tolerance of
the oracle's whole layer. The ranks run one after another on one GPU here (a
rank's forward waits on nothing another rank does).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_matmul_int8_b200 import _lib
from bit_quantized_matmul_int8_b200 import workloads as wl
from bit_quantized_matmul_int8_b200.shard import shard_rows
from gpu_common import case_inputs, check_y, dev, ensure_built, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def slice_codes(CB: torch.Tensor, N: int, K: int, n0: int, n1: int) -> torch.Tensor:
    """Rows [n0, n1) of blocked weight codes (n0 a multiple of 32): whole row blocks."""
    assert n0 % 32 == 0
    blocks = CB.view(-(-N // 32), -(-K // 128), 32, 128)
    return blocks[n0 // 32: -(-n1 // 32)].contiguous()


CASES = [
    # (M, K, N, outlier columns): decode GEMV, prefill GEMM with ragged tiles
    (4, 1024, 520, 5),
    (300, 1024, 520, 5),
    (77, 4096, 1032, 3),
]


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("M,K,N,n_out", CASES)
def test_shards_stitch_to_the_whole_layer(M, K, N, n_out, world):
    w = wl.random_case(300 + M + world, M, K, N, n_outliers=n_out, frac=0.5)
    X, W, b = case_inputs(w)
    Xd, Wd, bd = dev(X), dev(W), dev(b)
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    Y_whole = _lib.int8lt_forward(Xd, CB, SCB, Wd, w.threshold, bd)
    parts = []
    for r in range(world):
        n0, n1 = shard_rows(N, world, r)
        if n1 == n0:
            continue                                   # a rank with no channels
        CBs = slice_codes(CB, N, K, n0, n1)
        # the slice is what preparing the shard's own rows gives
        CBp, SCBp = _lib.int8lt_prepare_weight(Wd[n0:n1].contiguous())
        assert torch.equal(CBs, CBp.view_as(CBs)) and torch.equal(SCB[n0:n1], SCBp)
        Ys = _lib.int8lt_forward(Xd, CBs, SCB[n0:n1].contiguous(), Wd[n0:n1].contiguous(),
                                 w.threshold, bd[n0:n1].contiguous())
        parts.append(Ys)
    Y = torch.cat(parts, dim=1)
    torch.cuda.synchronize()
    assert Y.shape == (M, N)
    assert torch.equal(Y, Y_whole)
    CBo, SCBo = oracle.prepare_weight(W)
    Y64, _, n = oracle.forward(X, CBo, SCBo, W, w.threshold, b)
    assert n == n_out
    check_y(host(Y), Y64, f"{world} shards")


def test_proj_prefill_over_eight_shards():
    """The 2048 x 4096 x 4096 projection prefill split over 8 ranks (512 channels
    each), as bench.py --split runs it: bit-identical to the whole layer."""
    w = wl.WORKLOADS["proj_prefill_2048x4096x4096"]
    X, W, b = case_inputs(w)
    Xd, Wd = dev(X), dev(W)
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    Y_whole = _lib.int8lt_forward(Xd, CB, SCB, Wd, w.threshold, None)
    parts = []
    for r in range(8):
        n0, n1 = shard_rows(w.N, 8, r)
        parts.append(_lib.int8lt_forward(Xd, slice_codes(CB, w.N, w.K, n0, n1),
                                         SCB[n0:n1].contiguous(), Wd[n0:n1].contiguous(),
                                         w.threshold, None))
    Y = torch.cat(parts, dim=1)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y_whole)
    rows = np.array([0, 777, 2047])
    CBo, SCBo = oracle.prepare_weight(W)
    Y64, _, _ = oracle.forward(X, CBo, SCBo, W, w.threshold, None, rows=rows)
    check_y(host(Y)[rows], Y64, "8 shards")
