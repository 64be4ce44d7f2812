"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Integer stages (outlier set, CA/SCA, CB/SCB, int32 accumulators) must be
bit-exact; the fp16 output must satisfy |dY| <= 2e-3 * max(1, |y|) against
the oracle's fp64 value. Shapes span several 128 x 256 tiles with ragged tails.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_matmul_int8_b200 import _lib
from bit_quantized_matmul_int8_b200 import workloads as wl
from gpu_common import case_inputs, check_y, dev, ensure_built, host, run_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def gemm_i32_gpu(A: np.ndarray, B: np.ndarray) -> torch.Tensor:
    """int32 A . B^T through the GEMM / GEMV, B packed into the blocked weight layout."""
    return _lib.int8lt_debug_gemm_i32(dev(A), _lib.int8lt_pack_weight(dev(B)), B.shape[0])


# ------------------------------------------------------------ weight prep --

@pytest.mark.parametrize("N,K", [(64, 64), (200, 4096), (24, 40), (8, 3), (513, 1000)])
def test_prepare_weight_bit_exact(N, K):
    w = wl.random_case(31, 4, K, N)
    W = wl.make_w(w)
    W[N // 2] = 0                                   # all-zero channel: scale 0
    CB, SCB = _lib.int8lt_prepare_weight(dev(W))
    CBo, SCBo = oracle.prepare_weight(W)
    assert np.array_equal(host(_lib.int8lt_unpack_weight(CB, N, K)), CBo)
    assert np.array_equal(host(SCB).view(np.uint32), SCBo.view(np.uint32))
    # the blocked layout's padding (rows past N, columns past K) holds zero codes
    assert torch.equal(_lib.int8lt_pack_weight(dev(CBo)), CB)


@pytest.mark.parametrize("N,K", [(8, 16), (40, 136), (96, 4096), (33, 7), (64, 250)])
def test_weight_layout_roundtrip(N, K):
    rng = np.random.default_rng(N * 1000 + K)
    rows = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    CB = _lib.int8lt_pack_weight(dev(rows))
    assert CB.numel() == _lib.int8lt_weight_bytes(N, K) == -(-N // 32) * -(-K // 128) * 4096
    blk = host(CB).reshape(-(-N // 32), -(-K // 128), 32, 128)
    for j, k in [(0, 0), (N - 1, K - 1), (N // 2, K // 3), (min(N - 1, 31), min(K - 1, 127))]:
        assert blk[j // 32, k // 128, j % 32, k % 128] == rows[j, k]
    full = np.zeros((blk.shape[0] * 32, blk.shape[1] * 128), np.int8)
    full[:N, :K] = rows
    assert np.array_equal(blk.transpose(0, 2, 1, 3).reshape(full.shape), full)
    assert np.array_equal(host(_lib.int8lt_unpack_weight(CB, N, K)), rows)


def test_prepare_weight_idempotent():
    W = dev(wl.make_w(wl.random_case(32, 4, 256, 96)))
    a = [t.clone() for t in _lib.int8lt_prepare_weight(W)]
    b = _lib.int8lt_prepare_weight(W)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ---------------------------------------------------------- quantize rows --

QCASES = [
    ("tiny", wl.WORKLOADS["tiny_16x64x64"], None),
    ("ragged", wl.random_case(41, 37, 96, 8, n_outliers=5, frac=0.3), None),
    ("wide", wl.random_case(42, 130, 4112, 8, n_outliers=9, frac=0.75), None),
    ("many_rows", wl.random_case(43, 3000, 256, 8, n_outliers=3, frac=0.01), None),
    ("no_outliers", wl.random_case(44, 64, 512, 8, n_outliers=0), None),
    # more rows than shared memory keeps at once: several rounds
    ("rounds", wl.random_case(45, 4000, 4096, 8, n_outliers=7, frac=0.5), None),
    # rows of K >= 8192 are quantized by a whole CTA each, in rounds
    ("long_rows", wl.random_case(46, 1000, 16384, 8, n_outliers=4, frac=0.75), None),
    # long rows, ragged vector count, a few rows per CTA (streamed, a row per CTA)
    ("long_ragged", wl.random_case(48, 610, 10256, 8, n_outliers=5, frac=0.4), None),
    # rows too long to keep in shared memory: read from X in both phases
    ("very_long_rows", wl.random_case(47, 20, 65536, 8, n_outliers=3, frac=0.5), None),
    # decode batches (M <= 16): column slices of one cluster, staged or not
    ("decode_one_row", wl.random_case(49, 1, 12288, 8, n_outliers=6, frac=1.0), None),
    ("decode_ragged", wl.random_case(50, 7, 4112, 8, n_outliers=9, frac=0.5), None),
    ("decode_full", wl.random_case(51, 16, 12288, 8, n_outliers=24, frac=0.75), None),
    ("decode_max_k", wl.random_case(52, 16, 133136, 8, n_outliers=5, frac=0.5), None),
]


@pytest.mark.parametrize("name,w,_", QCASES, ids=[c[0] for c in QCASES])
@pytest.mark.parametrize("thr", [None, math.inf, 0.0, 1.5])
def test_quantize_rows_bit_exact(name, w, _, thr):
    X = wl.make_x(w)
    t = w.threshold if thr is None else thr
    CA, SCA, idx = _lib.int8lt_quantize_rows(dev(X), t)
    CAo, SCAo, idxo = oracle.quantize_rows(X, t)
    assert np.array_equal(host(idx), idxo)
    assert np.array_equal(host(CA), CAo)
    assert np.array_equal(host(SCA).view(np.uint32), SCAo.view(np.uint32))
    if thr is None:
        assert host(idx).tolist() == wl.outlier_columns(w).tolist()


@pytest.mark.parametrize("M,K", [(40, 256), (300, 1040), (2048, 4096), (17, 4096), (40, 8192), (33, 8208),
                                 (300, 16384), (700, 12288), (7, 64), (16, 12288), (9, 133136)])
def test_quantize_row_max_in_other_rows_outlier_column(M, K):
    """A row whose largest magnitude sits in a column that only other rows make an
    outlier: its scale must come from the columns outside O (a ([P] decomposition)
    case where a row cannot decide its own scale before the batch's O is known)."""
    rng = np.random.default_rng(M + K)
    X = np.clip(rng.standard_normal((M, K)) * 0.5, -2.5, 2.5).astype(np.float16)
    X[0, 7] = 10.0                  # column 7 is an outlier column (row 0)
    X[1, 7] = 5.5                   # row 1's max, below the threshold, in column 7
    X[2, 7] = -5.9                  # row 2's max, negative
    X[3, 7] = 3.0                   # row 3: its max is tied between column 7 and 20
    X[3, 20] = 3.0
    X[4, :] = 0.0
    X[4, 7] = 1.0                   # row 4: its only non-zero is in O -> scale 0
    X[5, K - 1] = 7.0               # another outlier column at the last position
    X[6, K - 1] = -4.0
    CA, SCA, idx = _lib.int8lt_quantize_rows(dev(X), 6.0)
    CAo, SCAo, idxo = oracle.quantize_rows(X, 6.0)
    assert host(idx).tolist() == idxo.tolist() == [7, K - 1]
    assert np.array_equal(host(SCA).view(np.uint32), SCAo.view(np.uint32))
    assert np.array_equal(host(CA), CAo)
    assert host(SCA)[4] == 0.0 and float(host(SCA)[1]) < 5.5


def test_quantize_threshold_boundary():
    X = np.zeros((40, 64), np.float16)
    X[3, 5] = 6.0
    X[7, 9] = np.float16(5.99609375)
    X[30, 60] = -6.0
    X[11, 33] = 65504.0
    X[:, 0] = np.linspace(-1, 1, 40)
    CA, SCA, idx = _lib.int8lt_quantize_rows(dev(X), 6.0)
    assert host(idx).tolist() == [5, 33, 60]
    CAo, SCAo, _ = oracle.quantize_rows(X, 6.0)
    assert np.array_equal(host(CA), CAo) and np.array_equal(host(SCA), SCAo)


def test_quantize_empty_batch():
    X = torch.empty((0, 64), dtype=torch.float16, device="cuda")
    CA, SCA, idx = _lib.int8lt_quantize_rows(X, 6.0)
    assert CA.shape == (0, 64) and len(idx) == 0


# ------------------------------------------------------------ int32 GEMM --

GEMM_SHAPES = [(128, 256, 128), (300, 520, 400), (129, 264, 4112), (1000, 776, 2048),
               (17, 8, 16), (1, 64, 64), (4, 1000, 512), (16, 4096, 1024), (3, 40, 48),
               (4, 38400, 256), (16, 8, 4096),
               # decode shapes whose row blocks are split between CTAs, with a
               # short last K segment and a partial last row block
               (5, 20000, 3008), (16, 9992, 2064)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_int32_bit_exact(M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    A = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
    B = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    if M > 2:
        A[1] = 127
        B[0] = -127 if N > 1 else B[0]
    C = host(gemm_i32_gpu(A, B))
    ref = A.astype(np.int64) @ B.astype(np.int64).T          # exact in int64
    assert np.array_equal(C.astype(np.int64), ref)


# Tile counts above the resident CTA-pair count and not a multiple of it: the
# last tiles are split between two pairs (head + tail with int32 partials).
SPLIT_SHAPES = [(1280, 4096, 512), (2048, 4096, 384), (2304, 4352, 1152)]


@pytest.fixture
def split_always():
    prev = _lib.int8lt_set_gemm_split(_lib.SPLIT_ALWAYS)
    yield
    _lib.int8lt_set_gemm_split(prev)


@pytest.mark.parametrize("M,N,K", SPLIT_SHAPES)
def test_gemm_int32_split_tiles_bit_exact(M, N, K, split_always):
    rng = np.random.default_rng(M + N + K)
    A = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
    B = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    C = host(gemm_i32_gpu(A, B))
    assert np.array_equal(C, oracle.gemm_i32(A, B))


def test_gemm_int32_split_auto_sampled_rows():
    # 4 x 19 = 76 tiles of 64 k-blocks: the default policy splits the last wave
    M, N, K = 1024, 4864, 8192
    rng = np.random.default_rng(76)
    A = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
    B = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    C = host(gemm_i32_gpu(A, B))
    rows = np.array([0, 1, 255, 256, 300, 511, 512, 700, 767, 768, 1000, 1023])
    assert np.array_equal(C[rows], oracle.gemm_i32(A[rows], B))


def test_gemm_int32_matches_oracle_routine():
    rng = np.random.default_rng(9)
    A = rng.integers(-127, 128, (200, 336), dtype=np.int64).astype(np.int8)
    B = rng.integers(-127, 128, (264, 336), dtype=np.int64).astype(np.int8)
    assert np.array_equal(host(gemm_i32_gpu(A, B)), oracle.gemm_i32(A, B))


@pytest.mark.parametrize("M", [1, 16, 300])
def test_cb_only_16_byte_aligned(M):
    """CB at an address that is 16- but not 32-byte aligned (the API's minimum): the
    decode GEMV then reads it with 16-byte loads; results equal the aligned case."""
    N, K = 264, 1040
    rng = np.random.default_rng(M)
    A = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
    B = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    CB = _lib.int8lt_pack_weight(dev(B))
    buf = torch.empty(CB.numel() + 32, dtype=torch.int8, device="cuda")
    assert buf.data_ptr() % 32 == 0
    CB16 = buf[16:16 + CB.numel()]
    CB16.copy_(CB.view(-1))
    assert CB16.data_ptr() % 32 == 16
    C = host(_lib.int8lt_debug_gemm_i32(dev(A), CB16, N))
    assert np.array_equal(C, oracle.gemm_i32(A, B))
    w = wl.random_case(65, M, K, N, n_outliers=3, frac=1.0)
    X, W, b = case_inputs(w)
    CBw, SCB = _lib.int8lt_prepare_weight(dev(W))
    CBw16 = buf[16:16 + CBw.numel()]
    CBw16.copy_(CBw.view(-1))
    Y1 = _lib.int8lt_forward(dev(X), CBw, SCB, dev(W), 6.0, dev(b))
    Y2 = _lib.int8lt_forward(dev(X), CBw16, SCB, dev(W), 6.0, dev(b))
    assert torch.equal(Y1, Y2)


def test_gemm_int32_extreme_k():
    # K near the int32 limit: 127 * 127 * K stays below 2^31
    K = 133136
    A = np.full((20, K), 127, np.int8)
    B = np.full((8, K), -127, np.int8)
    C = host(gemm_i32_gpu(A, B))
    assert (C.astype(np.int64) == -127 * 127 * K).all()


# --------------------------------------------------------------- forward --

FCASES = [
    wl.WORKLOADS["tiny_16x64x64"],
    wl.random_case(51, 300, 512, 264, n_outliers=4, frac=0.5),
    wl.random_case(52, 129, 1040, 520, n_outliers=7, frac=0.75, has_bias=False),
    wl.random_case(53, 17, 256, 40, n_outliers=2),             # smallest prefill M
    wl.random_case(54, 1, 1024, 2048, n_outliers=3, frac=1.0),  # decode
    wl.random_case(55, 4, 768, 312, n_outliers=6, frac=1.0),
    wl.random_case(56, 16, 4096, 1024, n_outliers=6, frac=1.0, has_bias=False),
    wl.random_case(57, 600, 2048, 1024, n_outliers=70, frac=0.2),  # > 64 outliers
    wl.random_case(58, 200, 384, 136, n_outliers=0),
    wl.random_case(63, 7, 3008, 20000, n_outliers=5, frac=1.0),   # decode, split row blocks
    wl.random_case(64, 300, 12288, 264, n_outliers=9, frac=0.3),  # long rows, streamed quantize
]


@pytest.mark.parametrize("w", FCASES, ids=[w.name for w in FCASES])
@pytest.mark.parametrize("thr", ["cfg", "inf"])
def test_forward_vs_oracle(w, thr):
    t = w.threshold if thr == "cfg" else math.inf
    X, W, b = case_inputs(w)
    Yg, Y64 = run_forward(X, W, b, t)
    check_y(Yg, Y64, w.name)


SPLIT_FCASES = [
    wl.random_case(59, 1280, 512, 4096, n_outliers=6, frac=0.5),
    wl.random_case(60, 2048, 384, 4096, n_outliers=45, frac=0.3),   # two outlier k-blocks
    wl.random_case(61, 1280, 640, 4096, n_outliers=0, has_bias=False),
]


@pytest.mark.parametrize("w", SPLIT_FCASES, ids=[w.name for w in SPLIT_FCASES])
def test_forward_split_tiles_vs_oracle(w, split_always):
    X, W, b = case_inputs(w)
    Yg, Y64 = run_forward(X, W, b, w.threshold)
    check_y(Yg, Y64, w.name)


def test_forward_split_auto_sampled_rows():
    w = wl.random_case(62, 1024, 8192, 4864, n_outliers=6, frac=0.5)
    X, W, b = case_inputs(w)
    rows = [0, 1, 255, 256, 511, 512, 767, 768, 900, 1023]
    Yg, Y64 = run_forward(X, W, b, w.threshold, rows=rows)
    check_y(Yg, Y64, w.name)


@pytest.mark.parametrize("w", [FCASES[1], FCASES[4], FCASES[7]], ids=lambda w: w.name)
def test_forward_int8_outlier_weights(w):
    """W_outlier = NULL: outlier weights come from CB * SCB / 127."""
    X, W, b = case_inputs(w)
    Yg, Y64 = run_forward(X, W, b, w.threshold, keep_w=False)
    check_y(Yg, Y64, w.name)


@pytest.mark.parametrize("M", [1, 16, 200])
def test_forward_all_columns_outlier(M):
    """threshold 0: every column is an outlier, the layer is an fp16 matmul."""
    w = wl.random_case(60 + M, M, 192, 136, n_outliers=2)
    X, W, b = case_inputs(w)
    X[X == 0] = np.float16(1e-3)
    Yg, Y64 = run_forward(X, W, b, 0.0)
    check_y(Yg, Y64, "all-outlier")
    ref = X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)
    check_y(Yg, ref, "all-outlier vs fp64 matmul")


def test_forward_deterministic_and_reuses_workspace():
    w = FCASES[1]
    X, W, b = case_inputs(w)
    Xd, Wd, bd = dev(X), dev(W), dev(b)
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    ws = _lib.workspace(w.M, w.N, w.K)
    y1 = _lib.int8lt_forward(Xd, CB, SCB, Wd, 6.0, bd, ws=ws).clone()
    # a call with a different outlier set in between must not leak into the next
    X2 = X.copy()
    X2[:, 7] = 50.0
    _lib.int8lt_forward(dev(X2), CB, SCB, Wd, 6.0, bd, ws=ws)
    y2 = _lib.int8lt_forward(Xd, CB, SCB, Wd, 6.0, bd, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert _lib.int8lt_read_device_status(ws) == 0


def test_forward_empty_batch():
    W = dev(wl.make_w(wl.random_case(70, 1, 64, 64)))
    CB, SCB = _lib.int8lt_prepare_weight(W)
    X = torch.empty((0, 64), dtype=torch.float16, device="cuda")
    Y = _lib.int8lt_forward(X, CB, SCB, W, 6.0)
    assert Y.shape == (0, 64)


def test_forward_on_side_stream():
    w = FCASES[1]
    X, W, b = case_inputs(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        Xd, Wd, bd = dev(X), dev(W), dev(b)
        CB, SCB = _lib.int8lt_prepare_weight(Wd, stream=s)
        Y = _lib.int8lt_forward(Xd, CB, SCB, Wd, 6.0, bd, stream=s)
    s.synchronize()
    CBo, SCBo = oracle.prepare_weight(W)
    Y64, _, _ = oracle.forward(X, CBo, SCBo, W, 6.0, b)
    check_y(host(Y), Y64, "side stream")


# ------------------------------------------------------- failure detection --

def test_bounded_wait_reports_timeout():
    ws = _lib.workspace(32, 64, 64)
    assert _lib.int8lt_read_device_status(ws) == 0
    _lib.int8lt_debug_wait_timeout(ws, 1_000_000)          # 1 ms, nothing arrives
    assert _lib.int8lt_read_device_status(ws) == _lib.STATUS_CODE["INT8LT_ERR_TIMEOUT"]
    assert _lib.int8lt_read_device_status(ws) == 0           # the read cleared it
    # the context is still usable
    X = dev(wl.make_x(wl.WORKLOADS["tiny_16x64x64"]))
    CA, SCA, idx = _lib.int8lt_quantize_rows(X, 6.0)
    torch.cuda.synchronize()
    assert len(idx) == 2


def test_grid_barrier_timeout_is_reported_and_recoverable():
    """The quantize pass's grid-barrier wait, run out on purpose (a launch that
    counts one block more than it has, 1 ms limit): the workspace status reports
    INT8LT_ERR_TIMEOUT once, and after int8lt_workspace_init the next forwards
    through the same workspace equal the ones before."""
    w = wl.random_case(72, 300, 1024, 256, n_outliers=3, frac=0.5)
    X, W, b = case_inputs(w)
    Xd, Wd, bd = dev(X), dev(W), dev(b)
    CB, SCB = _lib.int8lt_prepare_weight(Wd)
    ws = _lib.workspace(w.M, w.N, w.K)
    ref = _lib.int8lt_forward(Xd, CB, SCB, Wd, 6.0, bd, ws=ws).clone()
    assert _lib.int8lt_read_device_status(ws) == 0
    _lib.int8lt_debug_barrier_timeout(ws, 1_000_000)
    assert _lib.int8lt_read_device_status(ws) == _lib.STATUS_CODE["INT8LT_ERR_TIMEOUT"]
    assert _lib.int8lt_read_device_status(ws) == 0           # the read cleared it
    _lib.int8lt_workspace_init(ws)
    for _ in range(2):
        Y = _lib.int8lt_forward(Xd, CB, SCB, Wd, 6.0, bd, ws=ws)
        torch.cuda.synchronize()
        assert torch.equal(Y, ref)
    assert _lib.int8lt_read_device_status(ws) == 0
    CBo, SCBo = oracle.prepare_weight(W)
    Y64, _, _ = oracle.forward(X, CBo, SCBo, W, 6.0, b)
    check_y(host(ref), Y64, "forward around the barrier timeout")


def test_workspace_shared_across_shapes():
    """One workspace, large enough for each call, serves calls of different
    shapes in turn (decode batches of several sizes, prefill batches of short
    rows and of long rows, whose pass hands rows out from a counter in the
    workspace, the zeropoint forward): each result equals the same call on a
    fresh workspace, twice in a row."""
    cases = [wl.random_case(74, 16, 4096, 1024, n_outliers=3, frac=1.0),
             wl.random_case(75, 4, 1024, 2056, n_outliers=2, frac=1.0),
             wl.random_case(76, 300, 1024, 1024, n_outliers=4, frac=0.5),
             wl.random_case(78, 2000, 8192, 256, n_outliers=5, frac=0.75),
             wl.random_case(79, 300, 12288, 520, n_outliers=2, frac=0.5),
             wl.random_case(77, 9, 4096, 1024, n_outliers=3, frac=1.0),
             wl.random_case(78, 2000, 8192, 256, n_outliers=5, frac=0.75),
             wl.random_case(74, 16, 4096, 1024, n_outliers=3, frac=1.0)]
    size = max(_lib.int8lt_workspace_size(c.M, c.N, c.K) for c in cases)
    shared = torch.empty(size, dtype=torch.uint8, device="cuda")
    _lib.int8lt_workspace_init(shared)
    for i, c in enumerate(cases):
        X, W, b = case_inputs(c)
        Xd, Wd, bd = dev(X), dev(W), dev(b)
        CB, SCB = _lib.int8lt_prepare_weight(Wd)
        ref = _lib.int8lt_forward(Xd, CB, SCB, Wd, 6.0, bd)
        for _ in range(2):
            Y = _lib.int8lt_forward(Xd, CB, SCB, Wd, 6.0, bd, ws=shared)
            torch.cuda.synchronize()
            assert torch.equal(Y, ref), (i, c.name)
        if c.M <= 16:   # the zeropoint decode forward on the same workspace
            CBz, NDB, ZB, SB = _lib.int8lt_prepare_weight_zp(Wd)
            refz = _lib.int8lt_forward_zp(Xd, CBz, NDB, ZB, SB, bd)
            Yz = _lib.int8lt_forward_zp(Xd, CBz, NDB, ZB, SB, bd, ws=shared)
            torch.cuda.synchronize()
            assert torch.equal(Yz, refz), (i, c.name, "zeropoint")
    assert _lib.int8lt_read_device_status(shared) == 0


def test_validation_errors_raise():
    W = dev(wl.make_w(wl.random_case(71, 1, 64, 64)))
    CB, SCB = _lib.int8lt_prepare_weight(W)
    X = dev(wl.make_x(wl.random_case(71, 32, 64, 64)))
    with pytest.raises(_lib.Int8ltError) as e:
        _lib.int8lt_forward(X, CB, SCB, W, float("nan"))
    assert e.value.name == "INT8LT_ERR_VALUE"
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.Int8ltError) as e:
        _lib.int8lt_forward(X, CB, SCB, W, 6.0, ws=ws)
    assert e.value.name == "INT8LT_ERR_WORKSPACE"


def test_split_halves_equal_forward():
    for w in (FCASES[1], FCASES[5]):
        X, W, b = case_inputs(w)
        Xd, Wd, bd = dev(X), dev(W), dev(b) if b is not None else None
        CB, SCB = _lib.int8lt_prepare_weight(Wd)
        y1 = _lib.int8lt_forward(Xd, CB, SCB, Wd, 6.0, bd)
        ws = _lib.workspace(w.M, w.N, w.K)
        y2 = torch.empty_like(y1)
        _lib.int8lt_forward_quantize(Xd, CB, SCB, Wd, 6.0, ws)
        _lib.int8lt_forward_matmul(w.M, w.K, CB, SCB, Wd, bd, y2, ws)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2)
