"""ctypes binding of libint8lt.so (include/int8lt.h).

Argument marshalling only: every step of the layer runs in the CUDA library.
torch supplies device memory and streams. There is no CPU fallback: if the
shared library is missing or the device is not a B200 (sm_100a), calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libint8lt.so")
# The same library built with -DINT8LT_DEBUG: its kernels check the index of
# every computed global access and report a failed check as INT8LT_ERR_BOUNDS.
CHECK_LIB_PATH = os.path.join(_HERE, "libint8lt_check.so")

STATUS = {
    0: "INT8LT_OK", 1: "INT8LT_ERR_NULL", 2: "INT8LT_ERR_SHAPE", 3: "INT8LT_ERR_ALIGN",
    4: "INT8LT_ERR_VALUE", 5: "INT8LT_ERR_WORKSPACE", 6: "INT8LT_ERR_CUDA",
    7: "INT8LT_ERR_TIMEOUT", 8: "INT8LT_ERR_UNSUPPORTED", 9: "INT8LT_ERR_TOO_LARGE",
    10: "INT8LT_ERR_BOUNDS",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}

# Every symbol include/int8lt.h declares.
EXPORTS = [
    "int8lt_status_string", "int8lt_version", "int8lt_workspace_size", "int8lt_workspace_init",
    "int8lt_read_device_status", "int8lt_prepare_weight", "int8lt_quantize_rows",
    "int8lt_forward", "int8lt_forward_quantize", "int8lt_forward_matmul",
    "int8lt_forward_static_scratch", "int8lt_static_scratch_read_status",
    "int8lt_debug_gemm_i32", "int8lt_debug_gemm_schedule", "int8lt_debug_tile_order",
    "int8lt_debug_wait_timeout",
    "int8lt_debug_barrier_timeout", "int8lt_debug_static_scratch_timeout", "int8lt_set_gemm_split",
    "int8lt_quantize_rows_zp", "int8lt_prepare_weight_zp", "int8lt_forward_zp",
    "int8lt_forward_zp_quantize", "int8lt_forward_zp_matmul",
    "int8lt_weight_bytes", "int8lt_pack_weight", "int8lt_unpack_weight", "int8lt_layer_bytes",
]


class Int8ltError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg}")
        self.status = status
        self.name = STATUS.get(status, "UNKNOWN")


_lock = threading.Lock()
_lib = None

_P, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_SIGS = {
    "int8lt_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "int8lt_version": (ctypes.c_int, []),
    "int8lt_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "int8lt_workspace_init": (ctypes.c_int, [_P, _SZ, _P]),
    "int8lt_read_device_status": (ctypes.c_int, [_P, _SZ, _P]),
    "int8lt_prepare_weight": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "int8lt_quantize_rows": (ctypes.c_int, [_P, _I64, _I64, _F, _P, _P, _P, _P, _P, _SZ, _P]),
    "int8lt_forward": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _F, _P, _P, _P, _SZ, _P]),
    "int8lt_forward_quantize": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _F, _P, _SZ, _P]),
    "int8lt_forward_matmul": (ctypes.c_int, [_I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "int8lt_forward_static_scratch": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _F, _P, _P, _P]),
    "int8lt_debug_gemm_i32": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "int8lt_static_scratch_read_status": (ctypes.c_int, [_P]),
    "int8lt_debug_wait_timeout": (ctypes.c_int, [_P, _SZ, _I64, _P]),
    "int8lt_debug_barrier_timeout": (ctypes.c_int, [_P, _SZ, _I64, _P]),
    "int8lt_debug_static_scratch_timeout": (ctypes.c_int, [_I64, _P]),
    "int8lt_debug_gemm_schedule": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, ctypes.c_int]),
    "int8lt_debug_tile_order": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P]),
    "int8lt_set_gemm_split": (ctypes.c_int, [ctypes.c_int]),
    "int8lt_quantize_rows_zp": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "int8lt_prepare_weight_zp": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "int8lt_forward_zp": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "int8lt_forward_zp_quantize": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _SZ, _P]),
    "int8lt_weight_bytes": (_SZ, [_I64, _I64]),
    "int8lt_layer_bytes": (_SZ, [_I64, _I64, ctypes.c_int]),
    "int8lt_pack_weight": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "int8lt_unpack_weight": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "int8lt_forward_zp_matmul": (ctypes.c_int, [_I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
}


def lib(path: str | None = None) -> ctypes.CDLL:
    """Load libint8lt.so (in-tree build); raises if it has not been built."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m bit_quantized_matmul_int8_b200.build`")
            _lib = _bind(ctypes.CDLL(LIB_PATH))
    return _lib


class using_library:
    """Context manager: route this module's calls to another build of the
    library (e.g. CHECK_LIB_PATH) inside the block; not for concurrent use."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        lib()                       # the regular library, loaded once
        with _lock:
            self.saved = _lib
            _lib = _bind(ctypes.CDLL(self.path))
        return _lib

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self.saved


def _bind(l: ctypes.CDLL) -> ctypes.CDLL:
    for name, (res, args) in _SIGS.items():
        f = getattr(l, name)
        f.restype = res
        f.argtypes = args
    return l


def _check(fn: str, st: int) -> None:
    if st != 0:
        raise Int8ltError(fn, st, lib().int8lt_status_string(st).decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype, name: str, shape=None, device=None, cuda: bool = True) -> None:
    """Check a tensor argument before it reaches the library: on a CUDA device
    (the same one as ``device`` when given), of ``dtype``, contiguous and, when
    ``shape`` is given, of exactly that shape."""
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the input on {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def forward_args(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                 W_outlier: torch.Tensor | None, bias: torch.Tensor | None,
                 Y: torch.Tensor | None, cuda: bool = True) -> tuple[int, int, int]:
    """Validate the tensors of a forward call and return (M, N, K).

    X fp16 [M, K]; SCB fp32 [N]; CB the blocked codes of an [N, K] weight;
    W_outlier fp16 [N, K] or None; bias fp16 [N] or None; Y fp16 [M, N] or
    None. Everything on X's device. Raises ValueError before any launch, so
    that a buffer of the wrong size never reaches a kernel.
    """
    if X.dim() != 2:
        raise ValueError(f"X must be 2-D [M, K], got shape {tuple(X.shape)}")
    M, K = X.shape
    _dev(X, torch.float16, "X", cuda=cuda)
    if SCB.dim() != 1:
        raise ValueError(f"SCB must be 1-D [N], got shape {tuple(SCB.shape)}")
    N = SCB.shape[0]
    _dev(SCB, torch.float32, "SCB", device=X.device, cuda=cuda)
    _dev(CB, torch.int8, "CB", device=X.device, cuda=cuda)
    if CB.numel() != int8lt_weight_bytes(N, K):
        raise ValueError(f"CB holds {CB.numel()} bytes; the blocked codes of a [{N},{K}] weight "
                         f"take {int8lt_weight_bytes(N, K)}")
    if W_outlier is not None:
        _dev(W_outlier, torch.float16, "W_outlier", (N, K), X.device, cuda)
    if bias is not None:
        _dev(bias, torch.float16, "bias", (N,), X.device, cuda)
    if Y is not None:
        _dev(Y, torch.float16, "Y", (M, N), X.device, cuda)
    return M, N, K


# ------------------------------------------------------------ entry points --

def int8lt_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().int8lt_workspace_size(M, N, K))


def int8lt_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check("int8lt_workspace_init",
           lib().int8lt_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))


def int8lt_read_device_status(ws: torch.Tensor, stream=None) -> int:
    """Status code (0 = OK, 7 = a kernel timed out); clears the status word."""
    return int(lib().int8lt_read_device_status(_ptr(ws), ws.numel(), _stream(stream)))


def workspace(M: int, N: int, K: int, device=None) -> torch.Tensor:
    """Allocate (uint8) and initialise a workspace for an [M,K] x [N,K]^T call."""
    n = int8lt_workspace_size(M, N, K)
    if n == 0:
        raise Int8ltError("int8lt_workspace_size", 2, f"unsupported shape M={M} N={N} K={K}")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    int8lt_workspace_init(ws)
    return ws


def blocked_weight(N: int, K: int, device=None) -> torch.Tensor:
    """Uninitialised int8 buffer for [N,K] weight codes in the blocked weight layout:
    shape [ceil(N/32), ceil(K/128), 32, 128] (row block, k-block, row, byte)."""
    return torch.empty(((N + 31) // 32, (K + 127) // 128, 32, 128), dtype=torch.int8,
                       device=device or "cuda")


def _check_cb(CB: torch.Tensor, N: int, K: int) -> None:
    _dev(CB, torch.int8, "CB")
    if CB.numel() != int8lt_weight_bytes(N, K):
        raise ValueError(f"CB holds {CB.numel()} bytes; the blocked codes of a [{N},{K}] weight "
                         f"take {int8lt_weight_bytes(N, K)}")


def int8lt_weight_bytes(N: int, K: int) -> int:
    return int(lib().int8lt_weight_bytes(N, K))


def int8lt_layer_bytes(N: int, K: int, keep_fp16_weight: bool) -> int:
    """Resident device bytes of a prepared [N,K] layer (CB + SCB [+ fp16 W])."""
    return int(lib().int8lt_layer_bytes(N, K, int(bool(keep_fp16_weight))))


def int8lt_pack_weight(CB_rows: torch.Tensor, stream=None) -> torch.Tensor:
    """Row-major int8 codes [N,K] -> the blocked weight layout."""
    _dev(CB_rows, torch.int8, "CB_rows")
    N, K = CB_rows.shape
    CB = blocked_weight(N, K, CB_rows.device)
    _check("int8lt_pack_weight",
           lib().int8lt_pack_weight(_ptr(CB_rows), N, K, _ptr(CB), _stream(stream)))
    return CB


def int8lt_unpack_weight(CB: torch.Tensor, N: int, K: int, stream=None) -> torch.Tensor:
    """Blocked weight codes -> row-major int8 [N,K]."""
    _check_cb(CB, N, K)
    rows = torch.empty((N, K), dtype=torch.int8, device=CB.device)
    _check("int8lt_unpack_weight",
           lib().int8lt_unpack_weight(_ptr(CB), N, K, _ptr(rows), _stream(stream)))
    return rows


def int8lt_prepare_weight(W: torch.Tensor, CB: torch.Tensor | None = None,
                          SCB: torch.Tensor | None = None, stream=None):
    """W fp16 [N,K] -> (CB int8, blocked weight layout, SCB fp32 [N])."""
    _dev(W, torch.float16, "W")
    N, K = W.shape
    CB = blocked_weight(N, K, W.device) if CB is None else CB
    _check_cb(CB, N, K)
    SCB = torch.empty(N, dtype=torch.float32, device=W.device) if SCB is None else SCB
    _check("int8lt_prepare_weight",
           lib().int8lt_prepare_weight(_ptr(W), N, K, _ptr(CB), _ptr(SCB), _stream(stream)))
    return CB, SCB


def int8lt_quantize_rows(X: torch.Tensor, threshold: float = 6.0, ws: torch.Tensor | None = None,
                         stream=None):
    """X fp16 [M,K] -> (CA int8 [M,K], SCA fp32 [M], outlier_idx int32 [|O|])."""
    _dev(X, torch.float16, "X")
    M, K = X.shape
    dev = X.device
    CA = torch.empty((M, K), dtype=torch.int8, device=dev)
    SCA = torch.empty(M, dtype=torch.float32, device=dev)
    idx = torch.empty(max(K, 1), dtype=torch.int32, device=dev)
    n = torch.zeros(1, dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(M, 8, K, dev)
    _check("int8lt_quantize_rows",
           lib().int8lt_quantize_rows(_ptr(X), M, K, float(threshold), _ptr(CA), _ptr(SCA),
                                      _ptr(idx), _ptr(n), _ptr(ws), ws.numel(), _stream(stream)))
    return CA, SCA, idx[: int(n.item())]


def int8lt_forward(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                   W_outlier: torch.Tensor | None, threshold: float = 6.0,
                   bias: torch.Tensor | None = None, Y: torch.Tensor | None = None,
                   ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y fp16 [M,N] = LLM.int8() forward of X fp16 [M,K] with CB/SCB (and fp16 outlier weights)."""
    M, N, K = forward_args(X, CB, SCB, W_outlier, bias, Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    if ws is None:
        ws = workspace(M, N, K, X.device)
    _check("int8lt_forward",
           lib().int8lt_forward(_ptr(X), M, N, K, _ptr(CB), _ptr(SCB), _ptr(W_outlier),
                                float(threshold), _ptr(bias), _ptr(Y), _ptr(ws), ws.numel(),
                                _stream(stream)))
    return Y


def int8lt_forward_quantize(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                            W_outlier: torch.Tensor | None, threshold: float, ws: torch.Tensor,
                            stream=None) -> None:
    """First half of int8lt_forward: quantize X (and gather outlier weights) into ws."""
    M, N, K = forward_args(X, CB, SCB, W_outlier, None, None)
    _check("int8lt_forward_quantize",
           lib().int8lt_forward_quantize(_ptr(X), M, N, K, _ptr(CB), _ptr(SCB), _ptr(W_outlier),
                                         float(threshold), _ptr(ws), ws.numel(), _stream(stream)))


def int8lt_forward_matmul(M: int, K: int, CB: torch.Tensor, SCB: torch.Tensor,
                          W_outlier: torch.Tensor | None, bias: torch.Tensor | None,
                          Y: torch.Tensor, ws: torch.Tensor, stream=None) -> torch.Tensor:
    """Second half of int8lt_forward: GEMM/GEMV + fused epilogue from ws into Y."""
    N = SCB.shape[0]
    _dev(Y, torch.float16, "Y", (M, N))
    _dev(SCB, torch.float32, "SCB", (N,), Y.device)
    _check_cb(CB, N, K)
    if W_outlier is not None:
        _dev(W_outlier, torch.float16, "W_outlier", (N, K), Y.device)
    if bias is not None:
        _dev(bias, torch.float16, "bias", (N,), Y.device)
    _check("int8lt_forward_matmul",
           lib().int8lt_forward_matmul(M, N, K, _ptr(CB), _ptr(SCB), _ptr(W_outlier), _ptr(bias),
                                       _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def int8lt_forward_static_scratch(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                                  W_outlier: torch.Tensor | None, Y: torch.Tensor,
                                  threshold: float = 6.0, bias: torch.Tensor | None = None,
                                  stream=None) -> torch.Tensor:
    """Decode-shape forward (M <= 16) whose scratch is the library's fixed device array.

    For callers that cannot hand the layer a workspace: nothing is allocated by the call.
    ``Y`` must be supplied (allocating it here would defeat the purpose). Calls that
    overlap on the GPU share the one array and race; order them on one stream.
    """
    M, N, K = forward_args(X, CB, SCB, W_outlier, bias, Y)
    _check("int8lt_forward_static_scratch",
           lib().int8lt_forward_static_scratch(_ptr(X), M, N, K, _ptr(CB), _ptr(SCB),
                                               _ptr(W_outlier), float(threshold), _ptr(bias),
                                               _ptr(Y), _stream(stream)))
    return Y


def int8lt_debug_gemm_i32(CA: torch.Tensor, CB: torch.Tensor, N: int, ws: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """int32 CA [M,K] . CB^T with CB in the blocked weight layout (see int8lt_pack_weight)."""
    _dev(CA, torch.int8, "CA")
    M, K = CA.shape
    _check_cb(CB, N, K)
    C = torch.empty((M, N), dtype=torch.int32, device=CA.device)
    if ws is None:
        ws = workspace(M, N, K, CA.device)
    _check("int8lt_debug_gemm_i32",
           lib().int8lt_debug_gemm_i32(_ptr(CA), _ptr(CB), M, N, K, _ptr(C), _ptr(ws), ws.numel(),
                                       _stream(stream)))
    return C


def int8lt_debug_wait_timeout(ws: torch.Tensor, limit_ns: int, stream=None) -> None:
    _check("int8lt_debug_wait_timeout",
           lib().int8lt_debug_wait_timeout(_ptr(ws), ws.numel(), int(limit_ns), _stream(stream)))


def int8lt_debug_barrier_timeout(ws: torch.Tensor, limit_ns: int, stream=None) -> None:
    _check("int8lt_debug_barrier_timeout",
           lib().int8lt_debug_barrier_timeout(_ptr(ws), ws.numel(), int(limit_ns), _stream(stream)))


def int8lt_static_scratch_read_status(stream=None) -> int:
    """Status of int8lt_forward_static_scratch on the current device (0 = OK,
    7 = a kernel timed out); clears it and restores the array after a timeout."""
    return int(lib().int8lt_static_scratch_read_status(_stream(stream)))


def int8lt_debug_static_scratch_timeout(limit_ns: int, stream=None) -> None:
    _check("int8lt_debug_static_scratch_timeout",
           lib().int8lt_debug_static_scratch_timeout(int(limit_ns), _stream(stream)))


def int8lt_quantize_rows_zp(X: torch.Tensor, stream=None):
    """Zeropoint quantization of each row of X fp16 [R,K] -> (Q int8 [R,K], ND fp32 [R],
    ZP int32 [R], SUM int32 [R])."""
    _dev(X, torch.float16, "X")
    R, K = X.shape
    dev = X.device
    Q = torch.empty((R, K), dtype=torch.int8, device=dev)
    ND = torch.empty(R, dtype=torch.float32, device=dev)
    ZP = torch.empty(R, dtype=torch.int32, device=dev)
    SUM = torch.empty(R, dtype=torch.int32, device=dev)
    _check("int8lt_quantize_rows_zp",
           lib().int8lt_quantize_rows_zp(_ptr(X), R, K, _ptr(Q), _ptr(ND), _ptr(ZP), _ptr(SUM),
                                         _stream(stream)))
    return Q, ND, ZP, SUM


def int8lt_prepare_weight_zp(W: torch.Tensor, stream=None):
    """W fp16 [N,K] -> (CB int8 in the blocked weight layout, NDB fp32 [N], ZB int32 [N],
    SB int32 [N])."""
    _dev(W, torch.float16, "W")
    N, K = W.shape
    dev = W.device
    CB = blocked_weight(N, K, dev)
    NDB = torch.empty(N, dtype=torch.float32, device=dev)
    ZB = torch.empty(N, dtype=torch.int32, device=dev)
    SB = torch.empty(N, dtype=torch.int32, device=dev)
    _check("int8lt_prepare_weight_zp",
           lib().int8lt_prepare_weight_zp(_ptr(W), N, K, _ptr(CB), _ptr(NDB), _ptr(ZB), _ptr(SB),
                                          _stream(stream)))
    return CB, NDB, ZB, SB


def int8lt_forward_zp(X: torch.Tensor, CB: torch.Tensor, NDB: torch.Tensor, ZB: torch.Tensor,
                      SB: torch.Tensor, bias: torch.Tensor | None = None,
                      Y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """Y fp16 [M,N]: zeropoint-quantized X times the zeropoint-quantized weight, plus bias."""
    M, N, K = forward_args(X, CB, NDB, None, bias, Y)
    _dev(ZB, torch.int32, "ZB", (N,), X.device)
    _dev(SB, torch.int32, "SB", (N,), X.device)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    if ws is None:
        ws = workspace(M, N, K, X.device)
    _check("int8lt_forward_zp",
           lib().int8lt_forward_zp(_ptr(X), M, N, K, _ptr(CB), _ptr(NDB), _ptr(ZB), _ptr(SB),
                                   _ptr(bias), _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def int8lt_forward_zp_quantize(X: torch.Tensor, N: int, ws: torch.Tensor, stream=None) -> None:
    """First half of int8lt_forward_zp: zeropoint-quantize X's rows into ws."""
    _dev(X, torch.float16, "X")
    M, K = X.shape
    _check("int8lt_forward_zp_quantize",
           lib().int8lt_forward_zp_quantize(_ptr(X), M, N, K, _ptr(ws), ws.numel(), _stream(stream)))


def int8lt_forward_zp_matmul(M: int, K: int, CB: torch.Tensor, NDB: torch.Tensor, ZB: torch.Tensor,
                             SB: torch.Tensor, bias: torch.Tensor | None, Y: torch.Tensor,
                             ws: torch.Tensor, stream=None) -> None:
    """Second half of int8lt_forward_zp: GEMM/GEMV with the zeropoint epilogue into Y."""
    N = NDB.shape[0]
    _dev(Y, torch.float16, "Y", (M, N))
    _dev(NDB, torch.float32, "NDB", (N,), Y.device)
    _dev(ZB, torch.int32, "ZB", (N,), Y.device)
    _dev(SB, torch.int32, "SB", (N,), Y.device)
    _check_cb(CB, N, K)
    if bias is not None:
        _dev(bias, torch.float16, "bias", (N,), Y.device)
    _check("int8lt_forward_zp_matmul",
           lib().int8lt_forward_zp_matmul(M, N, K, _ptr(CB), _ptr(NDB), _ptr(ZB), _ptr(SB),
                                          _ptr(bias), _ptr(Y), _ptr(ws), ws.numel(),
                                          _stream(stream)))


SPLIT_AUTO, SPLIT_ALWAYS, SPLIT_NEVER = 0, 1, 2


def int8lt_set_gemm_split(mode: int) -> int:
    """Set the prefill GEMM's split policy (SPLIT_*); returns the previous one."""
    prev = int(lib().int8lt_set_gemm_split(int(mode)))
    if prev < 0:
        raise ValueError(f"unknown split mode {mode}")
    return prev


class Int8Linear:
    """LLM.int8() linear layer: Y = X W^T + bias with outlier decomposition.

    The counterpart of the Hugging Face ``Linear8bitLt(..., has_fp16_weights=False,
    threshold=6.0)``: the fp16 weight is converted once (``int8lt_prepare_weight``) and
    the forward runs ``int8lt_forward``. ``keep_fp16_outlier_weights=False`` drops the
    fp16 weight and takes the outlier columns' weights from CB * SCB / 127.
    """

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None = None,
                 threshold: float = 6.0, keep_fp16_outlier_weights: bool = True):
        self.N, self.K = weight.shape
        self.threshold = float(threshold)
        self.CB, self.SCB = int8lt_prepare_weight(weight.contiguous())
        self.W_outlier = weight.contiguous() if keep_fp16_outlier_weights else None
        self.bias = bias
        self._ws: dict[int, torch.Tensor] = {}

    def workspace_for(self, M: int, device) -> torch.Tensor:
        ws = self._ws.get(M)
        if ws is None:
            ws = self._ws[M] = workspace(M, self.N, self.K, device)
        return ws

    def __call__(self, X: torch.Tensor, Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        ws = self.workspace_for(X.shape[0], X.device)
        return int8lt_forward(X, self.CB, self.SCB, self.W_outlier, self.threshold, self.bias,
                              Y, ws, stream)
