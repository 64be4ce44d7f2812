"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` takes an oracle library handle (``oracle.load()`` or a mutant
built by the mutation test) and raises AssertionError when the oracle
disagrees with:

* the absmax worked example printed on the Hugging Face LLM.int8() page
  (``tests/golden/absmax_worked_example.txt``);
* the IEEE binary16 definition (numpy's own fp16 conversion over every bit
  pattern / many doubles);
* the weight recovery identity W ~= CB * SCB / 127 (Hugging Face page,
  "transformers integration") within half a quantization step;
* numpy's int64 matmul for the int8 GEMM (exact);
* brute-force column search for the outlier set, and the planted set;
* the decomposition equation's two special cases (LLM.int8() summary,
  "Mixed-precision Decomposition"): every column an outlier gives the fp64
  matmul X W^T + bias exactly (up to fp64 rounding); and
* a brute-force fp64 X W^T within the analytic quantization error bound;
* for zeropoint quantization (LLM.int8() summary, "8-bit Data Types and
  Quantization"): the row minimum maps to -127 and the maximum to 127, each
  element is rebuilt within half a step, the unrolled product equals the
  direct product of the shifted codes, and the forward stays within the
  quantization error bound.
"""
from __future__ import annotations

import math
import os

import numpy as np

import oracle
from bit_quantized_matmul_int8_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = [float(v) for v in vals]
    return out


# ------------------------------------------------------------------ fp16 --

def pin_half_decode(lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([lib.oracle_half_to_double(int(b)) for b in bits])
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin]), "binary16 decode differs from IEEE"
    assert np.isnan(got[~fin]).all()


def pin_half_encode(lib):
    rng = np.random.default_rng(7)
    vals = [0.0, -0.0, 1.0, 65504.0, 65519.99, 65520.0, 1e9, 2.0 ** -24, 2.0 ** -25,
            3 * 2.0 ** -25, 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25,
            1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2048 + 1.0, 2048 + 3.0, -5.4, 6.0, 5.99]
    vals += list(rng.standard_normal(3000) * 10.0 ** rng.integers(-9, 5, 3000))
    # exact ties between adjacent fp16 values
    h = rng.integers(0, 0x7bff, 2000).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    vals += list((lo + hi) / 2)
    for v in vals:
        with np.errstate(over="ignore"):
            ref = int(np.array([v], dtype=np.float64).astype(np.float16).view(np.uint16)[0])
        got = int(lib.oracle_double_to_half(float(v)))
        assert got == ref, f"binary16 encode of {v!r}: {got:#06x} != {ref:#06x}"


# ------------------------------------------------------- absmax quantize --

def pin_worked_example(lib):
    g = read_golden("absmax_worked_example.txt")
    x = np.array([g["values"]], dtype=np.float16)
    CA, SCA, idx = oracle.quantize_rows(x, math.inf, lib=lib)
    assert len(idx) == 0
    assert abs(127.0 / float(SCA[0]) - g["scale"][0]) <= g["scale_tolerance"][0]
    assert CA[0].tolist() == [int(c) for c in g["codes"]], CA[0].tolist()
    # the same vector as a weight row (per output channel)
    CB, SCB = oracle.prepare_weight(x, lib=lib)
    assert CB[0].tolist() == [int(c) for c in g["codes"]]
    assert float(SCB[0]) == float(np.float16(5.4))


def pin_absmax_invariants(lib):
    rng = np.random.default_rng(1)
    X = (rng.standard_normal((40, 97)) * rng.uniform(0.01, 5, (40, 1))).astype(np.float16)
    X[3] = 0.0                                  # all-zero row: scale 0, codes 0
    CA, SCA, _ = oracle.quantize_rows(X, math.inf, lib=lib)
    Xf = X.astype(np.float64)
    a = np.abs(Xf).max(axis=1)
    assert np.array_equal(SCA.astype(np.float64), a), "row scale must be the row absmax"
    assert np.abs(CA.astype(np.int32)).max() <= 127
    for i in range(X.shape[0]):
        if a[i] == 0:
            assert not CA[i].any()
            continue
        j = int(np.argmax(np.abs(Xf[i])))
        assert abs(int(CA[i, j])) == 127 and np.sign(CA[i, j]) == np.sign(Xf[i, j])
        err = np.abs(Xf[i] - CA[i].astype(np.float64) * a[i] / 127.0)
        assert (err <= a[i] / 254.0 * (1 + 1e-5)).all(), "error above half a step"


def pin_weight_recovery(lib):
    w = wl.WORKLOADS["tiny_16x64x64"].with_(N=48, K=80)
    W = wl.make_w(w)
    CB, SCB = oracle.prepare_weight(W, lib=lib)
    Wf = W.astype(np.float64)
    assert np.array_equal(SCB.astype(np.float64), np.abs(Wf).max(axis=1))
    rec = CB.astype(np.float64) * SCB[:, None].astype(np.float64) / 127.0
    assert (np.abs(Wf - rec) <= SCB[:, None] / 254.0 * (1 + 1e-5)).all()
    assert np.abs(CB.astype(np.int32)).max() == 127


# ------------------------------------------------------------ outlier set --

def pin_outlier_bruteforce(lib):
    rng = np.random.default_rng(3)
    X = (rng.standard_normal((9, 33)) * 3).astype(np.float16)
    for thr in (0.5, 4.0, 6.0, 7.5):
        want = [h for h in range(33) if any(abs(float(X[i, h])) >= thr for i in range(9))]
        assert oracle.outlier_columns(X, thr, lib=lib).tolist() == want


def pin_outlier_boundary(lib):
    X = np.zeros((3, 8), dtype=np.float16)
    X[0, 1] = 6.0                      # exactly the threshold: an outlier (|x| >= 6)
    X[1, 2] = np.float16(5.99609375)   # largest fp16 below 6: not an outlier
    X[2, 5] = -6.0                     # magnitude counts, not sign
    X[1, 7] = 65504.0
    assert oracle.outlier_columns(X, 6.0, lib=lib).tolist() == [1, 5, 7]
    assert oracle.outlier_columns(X, math.inf, lib=lib).tolist() == []
    assert oracle.outlier_columns(X, 0.0, lib=lib).tolist() == list(range(8))


def pin_planted_outliers(lib):
    for name in ("tiny_16x64x64",):
        w = wl.WORKLOADS[name]
        X = wl.make_x(w)
        got = oracle.outlier_columns(X, w.threshold, lib=lib)
        assert got.tolist() == wl.outlier_columns(w).tolist()


def pin_row_scale_excludes_outliers(lib):
    X = np.array([[0.5, 30.0, -2.0, 1.0],
                  [0.25, 1.0, 0.125, -0.5]], dtype=np.float16)
    CA, SCA, idx = oracle.quantize_rows(X, 6.0, lib=lib)
    assert idx.tolist() == [1]
    assert SCA.tolist() == [2.0, 0.5]                 # absmax over columns 0, 2, 3
    assert CA[:, 1].tolist() == [0, 0]                # outlier column is zero in CA
    assert CA[0].tolist() == [32, 0, -127, 64]        # 0.5*63.5=31.75 -> 32, 1*63.5=63.5 -> 64
    assert CA[1].tolist() == [64, 0, 32, -127]        # 0.25*254=63.5 -> 64


def pin_round_ties_to_even(lib):
    # absmax 127/64 makes the scale exactly 64, so x = (2k+1)/128 lands on k + 0.5
    X = np.array([[1.984375, 0.5078125, -0.5078125, 0.5234375, 0.0]], dtype=np.float16)
    CA, SCA, _ = oracle.quantize_rows(X, math.inf, lib=lib)
    assert 127.0 / float(SCA[0]) == 64.0
    assert CA[0].tolist() == [127, 32, -32, 34, 0]    # 32.5 -> 32, -32.5 -> -32, 33.5 -> 34


# -------------------------------------------------------------- int GEMM --

def pin_gemm_exact(lib):
    rng = np.random.default_rng(5)
    for (M, N, K) in [(1, 1, 1), (7, 5, 33), (16, 24, 300)]:
        A = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
        B = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
        ref = A.astype(np.int64) @ B.astype(np.int64).T
        assert np.array_equal(oracle.gemm_i32(A, B, lib=lib).astype(np.int64), ref)
    K = 4099
    A = np.full((2, K), 127, np.int8)
    B = np.full((3, K), -127, np.int8)
    assert (oracle.gemm_i32(A, B, lib=lib) == -127 * 127 * K).all()


def pin_gemm_overflow(lib):
    K = 133200                                    # 127^2 * K > 2^31 - 1
    A = np.full((1, K), 127, np.int8)
    try:
        oracle.gemm_i32(A, A, lib=lib)
    except OverflowError:
        return
    raise AssertionError("int32 overflow not reported")


# ------------------------------------------------------- whole forward ----

def _inputs(w, cut=None):
    X = wl.make_x(w, background_threshold=cut)
    W = wl.make_w(w)
    b = wl.make_bias(w)
    return X, W, b


def pin_all_columns_outlier(lib):
    """Decomposition eq. with O = every column: the fp16 product only."""
    for w in (wl.WORKLOADS["tiny_16x64x64"], wl.random_case(11, 13, 40, 24)):
        X, W, b = _inputs(w)
        CB, SCB = oracle.prepare_weight(W, lib=lib)
        Y64, Y16, n = oracle.forward(X, CB, SCB, W, 0.0, b, lib=lib)
        assert n == w.K
        ref = X.astype(np.float64) @ W.astype(np.float64).T
        if b is not None:
            ref += b.astype(np.float64)
        assert np.allclose(Y64, ref, rtol=1e-12, atol=1e-12), np.abs(Y64 - ref).max()
        assert np.array_equal(Y16, ref.astype(np.float16))


def pin_all_columns_outlier_int8_weights(lib):
    """O = every column and no fp16 weight kept: the product with CB*SCB/127."""
    w = wl.random_case(12, 9, 48, 20)
    X, W, b = _inputs(w)
    CB, SCB = oracle.prepare_weight(W, lib=lib)
    Y64, _, n = oracle.forward(X, CB, SCB, None, 0.0, b, lib=lib)
    rec = CB.astype(np.float64) * SCB[:, None].astype(np.float64) / 127.0
    Xf = X.astype(np.float64)
    ref = Xf @ rec.T + b.astype(np.float64)
    # each recovered weight is rounded to fp16 once: relative half-ulp 2^-11
    tol = np.abs(Xf) @ np.abs(rec).T * 2.0 ** -11 * (1 + 1e-6) + 1e-12
    assert (np.abs(Y64 - ref) <= tol).all()
    Wo = oracle.outlier_weights(None, CB, SCB, np.arange(w.K, dtype=np.int32), lib=lib)
    assert (np.abs(Wo.astype(np.float64) - W.astype(np.float64))
            <= SCB[:, None] / 254.0 + np.abs(rec) * 2.0 ** -11 + 1e-12).all()


def pin_outlier_weight_gather(lib):
    w = wl.random_case(13, 4, 64, 10)
    W = wl.make_w(w)
    CB, SCB = oracle.prepare_weight(W, lib=lib)
    idx = np.array([0, 7, 63], np.int32)
    assert np.array_equal(oracle.outlier_weights(W, CB, SCB, idx, lib=lib), W[:, idx])


def quant_error_bound(X, W, SCA, SCB, O):
    """|Y - X W^T| <= sum_{h not in O} (|x| SCB/254 + |w| SCA/254 + SCA SCB/254^2)."""
    mask = np.ones(X.shape[1], bool)
    mask[O] = False
    xs = np.abs(X.astype(np.float64))[:, mask].sum(axis=1)[:, None]
    ws = np.abs(W.astype(np.float64))[:, mask].sum(axis=1)[None, :]
    sa = SCA.astype(np.float64)[:, None]
    sb = SCB.astype(np.float64)[None, :]
    return xs * sb / 254 + sa * ws / 254 + mask.sum() * sa * sb / 254 ** 2


def pin_forward_within_bound(lib):
    cases = [wl.WORKLOADS["tiny_16x64x64"],
             wl.random_case(21, 37, 96, 40, n_outliers=4, frac=0.3),
             wl.random_case(22, 5, 160, 72, n_outliers=0)]
    for w in cases:
        for thr in (w.threshold, math.inf):
            X, W, b = _inputs(w)
            CB, SCB = oracle.prepare_weight(W, lib=lib)
            Y64, Y16, n = oracle.forward(X, CB, SCB, W, thr, b, lib=lib)
            CA, SCA, O = oracle.quantize_rows(X, thr, lib=lib)
            want_O = wl.outlier_columns(w) if math.isfinite(thr) else np.zeros(0, int)
            assert O.tolist() == want_O.tolist() and n == len(O)
            ref = X.astype(np.float64) @ W.astype(np.float64).T
            if b is not None:
                ref += b.astype(np.float64)
            bound = quant_error_bound(X, W, SCA, SCB, O)
            err = np.abs(Y64 - ref)
            assert (err <= bound * (1 + 1e-4) + 1e-9).all(), (w.name, thr, (err - bound).max())
            # The int8 part alone, where there is one, is a real correction term:
            # the error is far below the magnitude of the outlier product.
            if len(O):
                Xo = X.astype(np.float64)[:, O]
                Wo = W.astype(np.float64)[:, O]
                assert np.abs(Xo @ Wo.T).max() > 20 * bound.max()
            assert np.array_equal(Y16, Y64.astype(np.float16))


def pin_row_subset(lib):
    """The oracle's forwards for a subset of rows (as the full-size parity tests
    and the CPU baseline call them) equal the matching rows of the whole-batch
    forward, for a non-contiguous, unsorted subset with a repeated row. The
    outlier set stays a property of the whole batch: a subset without any
    outlier row still gets the outlier product of the planted columns."""
    w = wl.random_case(31, 23, 80, 24, n_outliers=3, frac=0.3)
    X, W, b = _inputs(w)
    CB, SCB = oracle.prepare_weight(W, lib=lib)
    S = np.array([17, 2, 9, 21, 2, 0, 13], dtype=np.int64)
    for thr in (w.threshold, math.inf):
        full64, full16, n_full = oracle.forward(X, CB, SCB, W, thr, b, lib=lib)
        sub64, sub16, n_sub = oracle.forward(X, CB, SCB, W, thr, b, rows=S, lib=lib)
        assert n_sub == n_full
        assert np.array_equal(sub64, full64[S]) and np.array_equal(sub16, full16[S])
    # rows that hold no outlier value: O still comes from every row of X
    O = wl.outlier_columns(w)
    quiet = np.flatnonzero((np.abs(X[:, O].astype(np.float32)) < w.threshold).all(axis=1))
    assert len(quiet) >= 2
    sub64, _, n_sub = oracle.forward(X, CB, SCB, W, w.threshold, b, rows=quiet[::-1].copy(), lib=lib)
    assert n_sub == len(O)
    full64, _, _ = oracle.forward(X, CB, SCB, W, w.threshold, b, lib=lib)
    assert np.array_equal(sub64, full64[quiet[::-1]])
    QB, NDB, ZB, SB = oracle.zp_quantize_rows(W, lib=lib)
    zfull = oracle.zp_forward(X, QB, NDB, ZB, SB, b, lib=lib)
    zsub = oracle.zp_forward(X, QB, NDB, ZB, SB, b, rows=S, lib=lib)
    assert np.array_equal(zsub, zfull[S])


def _zp_rows(seed):
    """Rows for the zeropoint pins: symmetric, one-sided (ReLU-like), shifted
    far from zero, constant and all-zero rows."""
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((12, 61)) * rng.uniform(0.05, 4, (12, 1))).astype(np.float16)
    X[1] = np.abs(X[1])                                    # ReLU output: one-sided
    X[2] = (rng.uniform(100.0, 101.0, 61)).astype(np.float16)   # far from zero
    X[3] = np.float16(2.5)                                 # constant row
    X[4] = 0.0                                             # all-zero row
    return X


def pin_zp_invariants(lib):
    """[P4 zeropoint quantization]: nd = 2*127 / (max - min) maps the row onto
    [-127, 127]: the minimum lands on -127, the maximum on 127 (or 126 when
    fp32 rounding of nd lands just short), and every element is rebuilt as
    (q + zp) / nd within half a step 0.5 / nd."""
    X = _zp_rows(3)
    Q, ND, ZP, SUM = oracle.zp_quantize_rows(X, lib=lib)
    Xf = X.astype(np.float64)
    assert np.abs(Q.astype(np.int32)).max() <= 127
    assert np.array_equal(SUM, Q.astype(np.int64).sum(axis=1))
    for i in range(X.shape[0]):
        mn, mx = Xf[i].min(), Xf[i].max()
        if mx == mn:                                       # constant row
            assert ND[i] == 1.0 and (Q[i] == -127).all()
            assert int(Q[i, 0]) + int(ZP[i]) == int(np.rint(mn))
            continue
        assert abs(float(ND[i]) * (mx - mn) - 254.0) < 254.0 * 1e-6
        assert int(Q[i, int(np.argmin(Xf[i]))]) == -127
        assert int(Q[i, int(np.argmax(Xf[i]))]) in (126, 127)
        rebuilt = (Q[i].astype(np.float64) + float(ZP[i])) / float(ND[i])
        assert (np.abs(Xf[i] - rebuilt) <= 0.5 / float(ND[i]) * (1 + 1e-5)).all(), i
    # the one-sided row uses codes on both sides of zero, unlike absmax
    assert Q[1].min() == -127 and Q[1].max() >= 126
    CA, _, _ = oracle.quantize_rows(X[1:2], math.inf, lib=lib)
    assert CA.min() >= 0


def pin_zp_unrolled_product(lib):
    """[P4]: the unrolled form A.B + zp_b sum(A) + zp_a sum(B) + K zp_a zp_b
    equals the direct product (A + zp_a).(B + zp_b) of the shifted codes."""
    rng = np.random.default_rng(4)
    X = (rng.standard_normal((7, 45)) + 0.7).astype(np.float16)
    W = (rng.standard_normal((9, 45)) * 0.05 - 0.01).astype(np.float16)
    b = (rng.standard_normal(9) * 0.1).astype(np.float16)
    QA, NDA, ZA, _ = oracle.zp_quantize_rows(X, lib=lib)
    QB, NDB, ZB, SB = oracle.zp_quantize_rows(W, lib=lib)
    Y = oracle.zp_forward(X, QB, NDB, ZB, SB, b, lib=lib)
    A = QA.astype(np.int64) + ZA.astype(np.int64)[:, None]
    B = QB.astype(np.int64) + ZB.astype(np.int64)[:, None]
    C = A @ B.T
    want = C.astype(np.float64) / (NDA.astype(np.float64)[:, None] * NDB.astype(np.float64)[None, :])
    want += b.astype(np.float64)[None, :]
    assert np.array_equal(Y, want)


def pin_zp_forward_within_bound(lib):
    """The zeropoint forward against the fp64 X W^T + bias, within the
    quantization error: per product |x w - x' w'| <= 0.5/nd_a |w| + |x'| 0.5/nd_b."""
    rng = np.random.default_rng(5)
    X = np.abs(rng.standard_normal((6, 80))).astype(np.float16)        # one-sided
    W = (rng.standard_normal((11, 80)) * 0.05).astype(np.float16)
    b = (rng.standard_normal(11) * 0.1).astype(np.float16)
    QA, NDA, ZA, _ = oracle.zp_quantize_rows(X, lib=lib)
    QB, NDB, ZB, SB = oracle.zp_quantize_rows(W, lib=lib)
    Y = oracle.zp_forward(X, QB, NDB, ZB, SB, b, lib=lib)
    Xf, Wf = X.astype(np.float64), W.astype(np.float64)
    ref = Xf @ Wf.T + b.astype(np.float64)
    ea = 0.5 / NDA.astype(np.float64)
    eb = 0.5 / NDB.astype(np.float64)
    bound = ea[:, None] * np.abs(Wf).sum(axis=1)[None, :] + \
        (np.abs(Xf).sum(axis=1) + ea * X.shape[1])[:, None] * eb[None, :]
    assert (np.abs(Y - ref) <= bound * (1 + 1e-6) + 1e-12).all()


def pin_zp_worked_examples(lib):
    """[HF] zero-point maps a range such as [-1, 1] onto [-127, 127]; [P4] nd and the
    zeropoint shift: four rows worked by hand (``tests/golden/zeropoint_worked_examples.txt``),
    including two ties that round to even."""
    with open(os.path.join(GOLDEN, "zeropoint_worked_examples.txt")) as f:
        rows = [ln.strip() for ln in f if ln.strip().startswith("row ")]
    assert len(rows) == 4
    for ln in rows:
        parts = [p.split() for p in ln[4:].split("|")]
        vals = np.array([float(v) for v in parts[0]], dtype=np.float16)[None, :]
        nd, zp, codes = float(parts[1][1]), int(parts[2][1]), [int(c) for c in parts[3][1:]]
        Q, ND, ZP, SUM = oracle.zp_quantize_rows(vals, lib=lib)
        assert Q[0].tolist() == codes, (ln, Q[0].tolist())
        assert int(ZP[0]) == zp and abs(float(ND[0]) - nd) <= 1e-5 * nd, ln
        assert int(SUM[0]) == sum(codes)


PINS = [pin_half_decode, pin_half_encode, pin_worked_example, pin_absmax_invariants,
        pin_weight_recovery, pin_outlier_bruteforce, pin_outlier_boundary,
        pin_planted_outliers, pin_row_scale_excludes_outliers, pin_round_ties_to_even, pin_gemm_exact,
        pin_gemm_overflow, pin_all_columns_outlier, pin_all_columns_outlier_int8_weights,
        pin_outlier_weight_gather, pin_forward_within_bound, pin_zp_invariants, pin_zp_unrolled_product,
        pin_zp_forward_within_bound, pin_zp_worked_examples, pin_row_subset]
