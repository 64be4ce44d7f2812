"""Seeded synthetic workloads for the LLM.int8() linear layer.

This module only draws input tensors. It holds none of the layer's arithmetic
(no quantization, no matmul) so that both the CUDA path and the CPU oracle can
consume the same bytes without sharing any of the method's code.

The shapes and statistics follow the LLM.int8() pages:

* "LLM.int8() paper summary" (kurtkim.github.io), Introduction and
  "Mixed-precision Decomposition": at 6.7B scale the outliers sit in about six
  feature dimensions and touch about 75% of the sequence positions; 13B has at
  most seven such dimensions.
* "Hugging Face LLM.int8() integration" (agentlenshq.com), the toy module
  ``Linear8bitLt(64, 64)`` and the threshold 6.0.

Recipe (the same for every workload):

* X background ~ N(0, 1), drawn in float32 and rounded to fp16 (round to
  nearest even); any background value whose fp16 magnitude is >= the
  threshold is redrawn, so the outlier column set is exactly the planted one.
* ``n_outliers`` distinct columns chosen by a seeded permutation of [0, K).
  In each, exactly ``round(frac * M)`` rows chosen by a seeded permutation get
  ``sign * U(lo, hi)`` with sign = +-1 equiprobable.
* W ~ N(0, sigma_w) in fp16, ``nn.Linear`` layout [N, K]; bias ~ N(0, 0.01)
  where the workload has one.

Every tensor has its own Philox stream keyed by (seed, workload id, tensor id),
so a tensor does not change when another one is added or resized.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

THRESHOLD = 6.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    n_outliers: int
    outlier_frac: float
    outlier_lo: float = 6.0
    outlier_hi: float = 60.0
    sigma_w: float = 0.02
    has_bias: bool = False
    threshold: float = THRESHOLD
    seed: int = 0
    wid: int = 0  # stream key of the workload family

    @property
    def ops(self) -> int:
        """2*M*N*K: the effective op count used for TOPS."""
        return 2 * self.M * self.N * self.K

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _qkv(n_out: int, thr: float) -> Workload:
    tag = "inf" if math.isinf(thr) else f"{thr:g}"
    return Workload(f"qkv_prefill_8192x12288x36864_o{n_out}_t{tag}", 8192, 12288, 36864,
                    n_out, 0.75, threshold=thr, wid=5)


WORKLOADS: dict[str, Workload] = {}
for _w in [
    Workload("tiny_16x64x64", 16, 64, 64, 2, 0.25, 6.0, 40.0, 0.05, True, wid=1),
    Workload("proj_prefill_2048x4096x4096", 2048, 4096, 4096, 6, 0.75, wid=2),
    Workload("ffn_up_4096x4096x16384", 4096, 4096, 16384, 6, 0.75, wid=3),
    Workload("ffn_down_4096x16384x4096", 4096, 16384, 4096, 12, 0.75, wid=33),
    Workload("decode_m1_12288x49152", 1, 12288, 49152, 6, 1.0, wid=4),
    Workload("decode_m4_12288x49152", 4, 12288, 49152, 6, 1.0, wid=4),
    Workload("decode_m16_12288x49152", 16, 12288, 49152, 6, 1.0, wid=4),
] + [_qkv(o, t) for o in (0, 6, 24, 246) for t in (6.0, math.inf)]:
    WORKLOADS[_w.name] = _w

# The workload the headline number is quoted on: the largest single-GPU
# configuration, the 175B-class fused QKV prefill with 6 outlier columns at
# the threshold 6.0.
HEADLINE = "qkv_prefill_8192x12288x36864_o6_t6"

# Reported beside the headline: the 4096-token FFN prefill pair (tensor-bound)
# and the decode GEMV sweep (HBM-bound).
TARGETS = ("ffn_up_4096x4096x16384", "ffn_down_4096x16384x4096", "decode_m1_12288x49152",
           "decode_m4_12288x49152", "decode_m16_12288x49152")

_T_X, _T_OUTCOLS, _T_OUTROWS, _T_OUTVAL, _T_W, _T_BIAS = range(6)


def _rng(w: Workload, tensor_id: int, extra: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([w.seed, w.wid, tensor_id, extra])
    return np.random.Generator(np.random.Philox(ss))


def outlier_columns(w: Workload) -> np.ndarray:
    """The planted outlier columns, sorted ascending (int64)."""
    if w.n_outliers == 0:
        return np.zeros(0, dtype=np.int64)
    perm = _rng(w, _T_OUTCOLS).permutation(w.K)
    return np.sort(perm[: w.n_outliers])


def make_x(w: Workload, background_threshold: float | None = None) -> np.ndarray:
    """Hidden states X [M, K] fp16 with the planted outlier columns.

    The background is redrawn wherever its fp16 magnitude reaches the cut, so
    no column outside the planted set holds a value >= the cut. The cut is the
    workload's threshold, except for a threshold of +inf (every value passes),
    where the default 6.0 cut keeps the data identical to the thresholded run.
    """
    cut = background_threshold
    if cut is None:
        cut = w.threshold if math.isfinite(w.threshold) else THRESHOLD
    g = _rng(w, _T_X)
    x = g.standard_normal((w.M, w.K), dtype=np.float32).astype(np.float16)
    bad = np.abs(x.astype(np.float32)) >= cut
    while bad.any():
        n = int(bad.sum())
        x[bad] = g.standard_normal(n, dtype=np.float32).astype(np.float16)
        bad = np.abs(x.astype(np.float32)) >= cut
    cols = outlier_columns(w)
    nrows = int(round(w.outlier_frac * w.M))
    for c_i, c in enumerate(cols):
        gr = _rng(w, _T_OUTROWS, c_i)
        rows = gr.permutation(w.M)[:nrows]
        gv = _rng(w, _T_OUTVAL, c_i)
        mag = gv.uniform(w.outlier_lo, w.outlier_hi, size=nrows)
        sign = np.where(gv.random(nrows) < 0.5, -1.0, 1.0)
        x[rows, c] = (sign * mag).astype(np.float16)
    return x


def make_w(w: Workload) -> np.ndarray:
    """Weight W [N, K] fp16 (nn.Linear layout), ~N(0, sigma_w)."""
    g = _rng(w, _T_W)
    out = np.empty((w.N, w.K), dtype=np.float16)
    step = max(1, (1 << 26) // max(1, w.K))
    for r0 in range(0, w.N, step):
        r1 = min(w.N, r0 + step)
        out[r0:r1] = (g.standard_normal((r1 - r0, w.K), dtype=np.float32)
                      * np.float32(w.sigma_w)).astype(np.float16)
    return out


def make_bias(w: Workload) -> np.ndarray | None:
    if not w.has_bias:
        return None
    g = _rng(w, _T_BIAS)
    return (g.standard_normal(w.N, dtype=np.float32) * np.float32(0.01)).astype(np.float16)


def make_inputs(w: Workload) -> dict:
    return {"X": make_x(w), "W": make_w(w), "bias": make_bias(w)}


def random_case(seed: int, M: int, K: int, N: int, n_outliers: int = 3,
                frac: float = 0.5, has_bias: bool = True,
                threshold: float = THRESHOLD, sigma_w: float = 0.05) -> Workload:
    """An ad-hoc workload for parity tests at arbitrary (ragged) shapes."""
    return Workload(f"case_s{seed}_{M}x{K}x{N}_o{n_outliers}", M, K, N, n_outliers, frac,
                    6.0, 40.0, sigma_w, has_bias, threshold, seed=seed, wid=1000)
