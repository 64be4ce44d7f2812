"""bench.py's multi-process logic on CPU: world_size 2 over gloo.

Each rank reports a different device time; every rank must see the maximum,
and the whole-job rate counts every rank's units over that slowest time.
The reference arm prints from rank 0 only.
"""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as tdist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world,
                             timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank            # rank 1 is the slow one
        m = bench.max_over_ranks(mine, "cpu")
        rate = bench.whole_job_rate(100.0, 4, world, m)
        q.put((rank, m, rate))
    finally:
        tdist.destroy_process_group()


def test_max_over_ranks_and_rate_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, rate in got:
        assert m == 15.0
        assert abs(rate - 100.0 * 4 * 2 / 0.015) < 1e-6


def test_single_process_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.whole_job_rate(10.0, 2, 1, 1000.0) == 20.0


def test_reference_arm_other_ranks_print_nothing(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload = "tiny_16x64x64"
        steps = 1
        warmup = 0
        out = None
        quant = "absmax"

    bench.run_reference(A, rank=1, world=2)
    assert capsys.readouterr().out == ""
    bench.run_reference(A, rank=0, world=2)
    line = capsys.readouterr().out.strip()
    assert line.startswith("{") and '"impl": "reference"' in line


def test_reference_arm_zeropoint(capsys):
    import json

    import bench

    class A:
        workload = "tiny_16x64x64"
        steps = 1
        warmup = 0
        out = None
        quant = "zeropoint"

    bench.run_reference(A, rank=0, world=1)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["config"]["quant"] == "zeropoint"
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_cpu_baseline_legs_all_modes():
    """bench.py's CPU-baseline leg for each quantization and weight mode."""
    sys.path.insert(0, ROOT)
    import bench
    from bit_quantized_matmul_int8_b200 import workloads as wl

    w = wl.WORKLOADS["tiny_16x64x64"]
    for quant, keep_w in (("absmax", True), ("absmax", False), ("zeropoint", False)):
        cb = bench.cpu_oracle_sample(w, 0.05, quant=quant, keep_w=keep_w)
        assert cb["kind"] == "oracle" and cb["value"] > 0 and 1 <= cb["rows"] <= w.M
        assert ("zeropoint" in cb["sample"]) == (quant == "zeropoint")
