"""Output-channel sharding on CPU: ranges, and world_size 2 over gloo.

The outlier set depends on X alone, so a layer split by output channel over
ranks computes, column for column, exactly what the whole layer computes.
The ranks here run the oracle on their shard (this is a test of the
sharding and gathering logic, not of the kernels) and all-gather over gloo.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_quantized_matmul_int8_b200.shard import shard_rows, shard_width  # noqa: E402


@pytest.mark.parametrize("N,world", [(4096, 2), (4096, 8), (264, 2), (264, 3), (49152, 8), (40, 4), (8, 2)])
def test_shard_ranges_cover_n(N, world):
    got = [shard_rows(N, world, r) for r in range(world)]
    assert got[0][0] == 0 and got[-1][1] == N
    for (a0, a1), (b0, b1) in zip(got, got[1:]):
        assert a1 == b0
    for n0, n1 in got:
        assert (n0 % 32 == 0 or n0 == N) and (n1 - n0) % 8 == 0 and 0 <= n1 - n0 <= shard_width(N, world)


def test_shard_rows_rejects_bad_requests():
    for args in [(64, 0, 0), (64, 2, 2), (64, 2, -1), (-8, 2, 0)]:
        with pytest.raises(ValueError):
            shard_rows(*args)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as tdist

    import oracle
    from bit_quantized_matmul_int8_b200 import workloads as wl
    from bit_quantized_matmul_int8_b200.shard import gather_shards, shard_rows

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world,
                             timeout=datetime.timedelta(seconds=60))
    try:
        w = wl.random_case(91, 40, 256, 264, n_outliers=4, frac=0.5)
        X, W, b = wl.make_x(w), wl.make_w(w), wl.make_bias(w)
        n0, n1 = shard_rows(w.N, world, rank)
        CB, SCB = oracle.prepare_weight(W[n0:n1])
        Y64, _, n_out = oracle.forward(X, CB, SCB, W[n0:n1], w.threshold, b[n0:n1])
        g = gather_shards(torch.from_numpy(np.ascontiguousarray(Y64)), w.N).numpy()
        if rank == 0:
            full = np.concatenate([g[r, :, : shard_rows(w.N, world, r)[1] - shard_rows(w.N, world, r)[0]]
                                   for r in range(world)], axis=1)
            CBf, SCBf = oracle.prepare_weight(W)
            Yf, _, nf = oracle.forward(X, CBf, SCBf, W, w.threshold, b)
            q.put((bool(np.array_equal(full, Yf)), int(n_out), int(nf)))
    finally:
        tdist.destroy_process_group()


def test_sharded_forward_equals_whole_layer_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    same, n_shard, n_full = q.get(timeout=10)
    assert same and n_shard == n_full == 4
