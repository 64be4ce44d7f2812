"""CPU oracle for the LLM.int8() linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA path never routes through it.

The arithmetic lives in ``int8lt_oracle.c`` (plain single-threaded C, fp64
for the floating-point combination); this module only compiles it with gcc
and marshals numpy arrays. fp16 arrays cross as their raw uint16 bit patterns.

Every function below is pinned by ``tests/test_oracle_pins.py`` (worked
example, closed forms, special cases that reduce to a library routine, brute
force within the analytic error bound). None is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "int8lt_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lock = threading.Lock()
_lib = None


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library; ``path`` loads a variant."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    lib.oracle_half_to_double.restype = ctypes.c_double
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_double_to_half.restype = ctypes.c_uint16
    lib.oracle_double_to_half.argtypes = [ctypes.c_double]
    lib.oracle_outlier_columns.restype = _I64
    lib.oracle_outlier_columns.argtypes = [_P, _I64, _I64, ctypes.c_float, _P]
    lib.oracle_quantize_rows.restype = _I64
    lib.oracle_quantize_rows.argtypes = [_P, _I64, _I64, ctypes.c_float, _P, _P, _P]
    lib.oracle_prepare_weight.restype = None
    lib.oracle_prepare_weight.argtypes = [_P, _I64, _I64, _P, _P]
    lib.oracle_gemm_i32.restype = ctypes.c_int
    lib.oracle_gemm_i32.argtypes = [_P, _P, _I64, _I64, _I64, _P]
    lib.oracle_forward_rows.restype = _I64
    lib.oracle_forward_rows.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P, ctypes.c_float,
                                        _P, _P, _I64, _P, _P]
    lib.oracle_outlier_weights.restype = None
    lib.oracle_outlier_weights.argtypes = [_P, _P, _P, _I64, _I64, _P, _I64, _P]
    lib.oracle_zp_quantize_rows.restype = None
    lib.oracle_zp_quantize_rows.argtypes = [_P, _I64, _I64, _P, _P, _P, _P]
    lib.oracle_zp_forward_rows.restype = None
    lib.oracle_zp_forward_rows.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _I64, _P]
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _h(a: np.ndarray | None) -> np.ndarray | None:
    """fp16 array -> contiguous uint16 view (raw bits)."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16
    return a


def half_to_double(bits: int, lib=None) -> float:
    return (lib or load()).oracle_half_to_double(int(bits))


def double_to_half(x: float, lib=None) -> int:
    return int((lib or load()).oracle_double_to_half(float(x)))


def outlier_columns(X: np.ndarray, threshold: float, lib=None) -> np.ndarray:
    lib = lib or load()
    x = _h(X)
    M, K = x.shape
    idx = np.zeros(max(K, 1), dtype=np.int32)
    n = lib.oracle_outlier_columns(_ptr(x), M, K, float(threshold), _ptr(idx))
    return idx[:n].copy()


def quantize_rows(X: np.ndarray, threshold: float, lib=None):
    """-> (CA int8 [M,K], SCA fp32 [M], outlier_idx int32 [|O|])."""
    lib = lib or load()
    x = _h(X)
    M, K = x.shape
    CA = np.zeros((M, K), dtype=np.int8)
    SCA = np.zeros(M, dtype=np.float32)
    idx = np.zeros(max(K, 1), dtype=np.int32)
    n = lib.oracle_quantize_rows(_ptr(x), M, K, float(threshold), _ptr(CA), _ptr(SCA), _ptr(idx))
    return CA, SCA, idx[:n].copy()


def prepare_weight(W: np.ndarray, lib=None):
    """-> (CB int8 [N,K], SCB fp32 [N])."""
    lib = lib or load()
    w = _h(W)
    N, K = w.shape
    CB = np.zeros((N, K), dtype=np.int8)
    SCB = np.zeros(N, dtype=np.float32)
    lib.oracle_prepare_weight(_ptr(w), N, K, _ptr(CB), _ptr(SCB))
    return CB, SCB


def gemm_i32(A: np.ndarray, B: np.ndarray, lib=None) -> np.ndarray:
    """C = A @ B.T with int32 result (raises if a sum leaves int32)."""
    lib = lib or load()
    A = np.ascontiguousarray(A, dtype=np.int8)
    B = np.ascontiguousarray(B, dtype=np.int8)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    C = np.zeros((M, N), dtype=np.int32)
    if lib.oracle_gemm_i32(_ptr(A), _ptr(B), M, N, K, _ptr(C)) != 0:
        raise OverflowError("int32 accumulator overflow")
    return C


def forward(X, CB, SCB, W_outlier, threshold, bias, rows=None, lib=None):
    """-> (Y64 fp64 [r,N], Y16 fp16 [r,N], n_outliers) for rows ``rows`` (default all)."""
    lib = lib or load()
    x = _h(X)
    M, K = x.shape
    CB = np.ascontiguousarray(CB, dtype=np.int8)
    SCB = np.ascontiguousarray(SCB, dtype=np.float32)
    N = CB.shape[0]
    wo = _h(W_outlier)
    b = _h(bias)
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    Y64 = np.zeros((len(rows), N), dtype=np.float64)
    Y16 = np.zeros((len(rows), N), dtype=np.uint16)
    n = lib.oracle_forward_rows(_ptr(x), M, N, K, _ptr(CB), _ptr(SCB), _ptr(wo),
                                float(threshold), _ptr(b), _ptr(rows), len(rows),
                                _ptr(Y64), _ptr(Y16))
    if n < 0:
        raise OverflowError("int32 accumulator overflow")
    return Y64, Y16.view(np.float16), int(n)


def outlier_weights(W_outlier, CB, SCB, idx, lib=None) -> np.ndarray:
    """Gathered fp16 outlier weights Wo [N, |O|] as the forward uses them."""
    lib = lib or load()
    CB = np.ascontiguousarray(CB, dtype=np.int8)
    SCB = np.ascontiguousarray(SCB, dtype=np.float32)
    N, K = CB.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    Wo = np.zeros((N, max(len(idx), 1)), dtype=np.uint16)
    lib.oracle_outlier_weights(_ptr(_h(W_outlier)), _ptr(CB), _ptr(SCB), N, K, _ptr(idx),
                               len(idx), _ptr(Wo))
    return Wo[:, : len(idx)].view(np.float16)


def zp_quantize_rows(X, lib=None):
    """Zeropoint quantization of each row: -> (codes int8 [R,K], nd fp32 [R], zp int32 [R], sum int32 [R])."""
    lib = lib or load()
    x = _h(X)
    R, K = x.shape
    Q = np.zeros((R, K), dtype=np.int8)
    ND = np.zeros(R, dtype=np.float32)
    ZP = np.zeros(R, dtype=np.int32)
    SUM = np.zeros(R, dtype=np.int32)
    lib.oracle_zp_quantize_rows(_ptr(x), R, K, _ptr(Q), _ptr(ND), _ptr(ZP), _ptr(SUM))
    return Q, ND, ZP, SUM


def zp_forward(X, CB, NDB, ZPB, SUMB, bias, rows=None, lib=None) -> np.ndarray:
    """Zeropoint forward (no outlier split) -> Y64 fp64 [r, N] for rows ``rows`` (default all)."""
    lib = lib or load()
    x = _h(X)
    M, K = x.shape
    CB = np.ascontiguousarray(CB, dtype=np.int8)
    N = CB.shape[0]
    NDB = np.ascontiguousarray(NDB, dtype=np.float32)
    ZPB = np.ascontiguousarray(ZPB, dtype=np.int32)
    SUMB = np.ascontiguousarray(SUMB, dtype=np.int32)
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    Y64 = np.zeros((len(rows), N), dtype=np.float64)
    lib.oracle_zp_forward_rows(_ptr(x), M, N, K, _ptr(CB), _ptr(NDB), _ptr(ZPB), _ptr(SUMB), _ptr(_h(bias)),
                               _ptr(rows), len(rows), _ptr(Y64))
    return Y64
