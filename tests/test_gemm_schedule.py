"""The prefill GEMM's tile schedule (data-parallel + stream-K) and tile order, on the CPU.

int8lt_debug_gemm_schedule enumerates, on the host, the exact segments the
kernel walks. Every (tile, k-block) must be computed exactly once; a split
tile has one head (from k-block 0, finishing the tile) in pair p and one
tail (to the last k-block, handing its int32 sums over) in pair p + 1; the
k-blocks per pair differ by at most one tile's worth in the data-parallel
part and by at most one k-block in the stream-K part.
"""
import numpy as np
import pytest

from bit_quantized_matmul_int8_b200 import _lib, build


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def schedule(L, tiles, nkb, pairs, mode=_lib.SPLIT_ALWAYS):
    n = L.int8lt_debug_gemm_schedule(tiles, nkb, pairs, mode, None, 0)
    out = np.zeros((max(n, 1), 6), np.int32)
    assert L.int8lt_debug_gemm_schedule(tiles, nkb, pairs, mode, out.ctypes.data, n) == n
    return out[:n]


@pytest.mark.parametrize("tiles,nkb,pairs", [
    (128, 32, 74),      # 2048 x 4096 x 4096 on 74 pairs: 1.73 waves
    (1024, 32, 74),     # 4096 x 4096 x 16384
    (256, 128, 74),     # 4096 x 16384 x 4096
    (1152, 96, 74),     # 8192 x 12288 x 36864
    (74, 32, 74), (148, 8, 74), (3, 5, 3), (1, 1, 1), (7, 1, 4), (10, 3, 4), (75, 2, 74),
])
def test_schedule_covers_every_kblock_once(L, tiles, nkb, pairs):
    s = schedule(L, tiles, nkb, pairs)
    cover = np.zeros((tiles, nkb), np.int32)
    for p, t, k0, k1, head, tail in s:
        assert 0 <= t < tiles and 0 <= k0 < k1 <= nkb
        cover[t, k0:k1] += 1
        assert head == (k0 == 0 and k1 < nkb)
        assert tail == (k0 > 0)
        if tail:
            assert k1 == nkb
    assert (cover == 1).all()
    heads = {t: p for p, t, k0, k1, h, tl in s if h}
    tails = {t: p for p, t, k0, k1, h, tl in s if tl}
    assert heads.keys() == tails.keys()
    for t in heads:
        assert tails[t] == heads[t] + 1
    # a pair owns at most one head, as its last segment, and at most one tail,
    # as the first segment of its stream-K range (after its whole tiles, whose
    # count is the same for every pair, so the tail is ready long before the
    # head of the previous pair needs it)
    for p in range(pairs):
        mine = s[s[:, 0] == p]
        if len(mine):
            assert mine[:-1, 4].sum() == 0 and mine[:, 5].sum() <= 1
            if mine[:, 5].any():
                k = int(np.nonzero(mine[:, 5])[0][0])
                assert (mine[k + 1:, 1] > mine[k, 1]).all()
                assert (mine[:k, 2] == 0).all() and (mine[:k, 3] == nkb).all()
    # balance: stream-K k-blocks per pair differ by at most one
    work = np.array([(s[s[:, 0] == p, 3] - s[s[:, 0] == p, 2]).sum() for p in range(pairs)])
    if tiles % pairs and tiles > pairs:
        assert work.max() - work.min() <= 1
    assert work.sum() == tiles * nkb


def test_bad_arguments(L):
    assert L.int8lt_debug_gemm_schedule(4, 0, 2, 0, None, 0) == -1
    assert L.int8lt_debug_gemm_schedule(4, 2, 0, 0, None, 0) == -1
    assert L.int8lt_debug_gemm_schedule(4, 2, 2, 3, None, 0) == -1


def _is_split(s):
    return bool(s[:, 5].any())


@pytest.mark.parametrize("tiles,nkb,pairs,want", [
    (76, 64, 74, True),     # 1024 x 4864 x 8192: 1.03 waves, the second nearly empty
    (256, 128, 74, True),   # 4096 x 4096 x 16384: saves 69 k-blocks per pair
    (128, 32, 74, False),   # 2048 x 4096 x 4096: saves under 9 k-blocks per pair
    (80, 32, 74, False),    # saves 29 k-blocks, below one 4096-deep tile
    (1024, 32, 74, False),
    (148, 32, 74, False),   # exact waves: nothing to split
])
def test_auto_policy(L, tiles, nkb, pairs, want):
    assert _is_split(schedule(L, tiles, nkb, pairs, _lib.SPLIT_AUTO)) == want
    assert not _is_split(schedule(L, tiles, nkb, pairs, _lib.SPLIT_NEVER))
    s_auto = schedule(L, tiles, nkb, pairs, _lib.SPLIT_AUTO)
    cover = np.zeros((tiles, nkb), np.int32)
    for p, t, k0, k1, h, tl in s_auto:
        cover[t, k0:k1] += 1
    assert (cover == 1).all()


def test_set_gemm_split_roundtrip(L):
    prev = _lib.int8lt_set_gemm_split(_lib.SPLIT_NEVER)
    try:
        assert _lib.int8lt_set_gemm_split(_lib.SPLIT_ALWAYS) == _lib.SPLIT_NEVER
        with pytest.raises(ValueError):
            _lib.int8lt_set_gemm_split(7)
    finally:
        _lib.int8lt_set_gemm_split(prev)


def tile_order(L, num_m, num_n):
    out = np.full((num_m * num_n, 2), -1, np.int32)
    assert L.int8lt_debug_tile_order(num_m, num_n, out.ctypes.data) == num_m * num_n
    return out


@pytest.mark.parametrize("num_m,num_n", [
    (8, 16),     # 2048 x 4096: one group of 8 tile rows, the former order
    (16, 64),    # 4096 x 16384
    (32, 144),   # 8192 x 36864: four groups
    (17, 3),     # a last group of one tile row
    (13, 5), (1, 1), (1, 7), (9, 1), (24, 2),
])
def test_tile_order_is_a_grouped_permutation(L, num_m, num_n):
    """Every output tile is visited once; tiles go in groups of 8 tile rows
    (the last group may be shorter), tile column by tile column inside a group,
    tile row fastest; a group is finished before the next one starts."""
    o = tile_order(L, num_m, num_n)
    seen = np.zeros((num_m, num_n), np.int32)
    for m, n in o:
        assert 0 <= m < num_m and 0 <= n < num_n
        seen[m, n] += 1
    assert (seen == 1).all()
    t = 0
    for g0 in range(0, num_m, 8):
        rows = min(8, num_m - g0)
        for n in range(num_n):
            for m in range(g0, g0 + rows):
                assert tuple(o[t]) == (m, n), (t, tuple(o[t]), (m, n))
                t += 1
    assert t == num_m * num_n


def test_tile_order_bad_arguments(L):
    out = np.zeros(2, np.int32)
    assert L.int8lt_debug_tile_order(0, 1, out.ctypes.data) == -1
    assert L.int8lt_debug_tile_order(1, 0, out.ctypes.data) == -1
    assert L.int8lt_debug_tile_order(1, 1, None) == -1
