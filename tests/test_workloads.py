"""The seeded input generator: determinism and the stated recipe (CPU only)."""
import math

import numpy as np

from bit_quantized_matmul_int8_b200 import workloads as wl


def test_deterministic_and_shapes():
    w = wl.WORKLOADS["tiny_16x64x64"]
    a, b = wl.make_inputs(w), wl.make_inputs(w)
    assert a["X"].shape == (16, 64) and a["W"].shape == (64, 64) and a["bias"].shape == (64,)
    for k in ("X", "W", "bias"):
        assert a[k].dtype == np.float16 and np.array_equal(a[k], b[k])


def test_planted_columns_and_rows():
    for w in (wl.WORKLOADS["tiny_16x64x64"], wl.random_case(3, 40, 256, 8, n_outliers=5, frac=0.75)):
        X = wl.make_x(w).astype(np.float32)
        cols = wl.outlier_columns(w)
        assert len(cols) == w.n_outliers == len(set(cols.tolist()))
        big = np.abs(X) >= w.threshold
        assert sorted(set(np.nonzero(big)[1].tolist())) == cols.tolist()
        for c in cols:
            n = int(big[:, c].sum())
            assert n == round(w.outlier_frac * w.M)
            assert np.abs(X[big[:, c], c]).max() <= w.outlier_hi + 0.1


def test_inf_threshold_keeps_data():
    w = wl.WORKLOADS["qkv_prefill_8192x12288x36864_o6_t6"].with_(M=64, K=512, N=8)
    w_inf = w.with_(threshold=math.inf)
    assert np.array_equal(wl.make_x(w), wl.make_x(w_inf))


def test_headline_and_configs():
    assert wl.HEADLINE in wl.WORKLOADS
    h = wl.WORKLOADS[wl.HEADLINE]
    # the largest single-GPU configuration: the fused QKV prefill at threshold 6.0
    assert (h.M, h.K, h.N, h.n_outliers, h.threshold) == (8192, 12288, 36864, 6, 6.0)
    assert h.ops == max(w.ops for w in wl.WORKLOADS.values())
    assert all(t in wl.WORKLOADS and t != wl.HEADLINE for t in wl.TARGETS)
    assert wl.WORKLOADS["ffn_down_4096x16384x4096"].n_outliers == 12
    assert wl.WORKLOADS["qkv_prefill_8192x12288x36864_o246_t6"].n_outliers == 246
