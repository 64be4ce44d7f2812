"""Benchmark of the LLM.int8() linear layer on B200.

A step is one int8lt_forward (outlier detect + row quantize + int8 tensor-core
GEMM with the fused dequantize / fp16 outlier product / bias epilogue). The
headline workload is the largest single-GPU configuration, the 175B-class
fused QKV prefill X fp16 [8192 x 12288] . W [36864 x 12288]^T with 6 outlier
feature columns at the threshold 6.0, unless --workload says otherwise.
Inputs are resident in HBM; several input sets rotate so that the bytes
touched between two uses of a set exceed the 126 MB L2.

Prints ONE JSON line (rank 0). Value = effective TOPS = 2*M*N*K per forward,
summed over ranks, over the max-over-ranks device time of the timed steps.
The timed steps replay CUDA graphs of up to 10 whole steps without event
nodes between kernels; each half is then timed alone over the same steps for
the per-kernel figures (phases_ms, roofline). The same measurement, without
the host-buffer loop, runs on the 4096-token FFN prefill pair and the decode
sweep (M = 1, 4, 16) and is reported under `targets`.
Multi-GPU: one process per GPU, each runs its own replica (independent
batches, no collective on the data path); NCCL only for the barrier and the
max-over-ranks time.

--impl reference times the CPU oracle (plain single-threaded C) on a bounded
sample of the same workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from bit_quantized_matmul_int8_b200 import workloads as wl  # noqa: E402

METRIC = "int8 mixed-precision linear effective TOPS & tokens/s; % of INT8 peak / HBM BW"
L2_BYTES = 126 * 1024 * 1024
INT8_PER_BF16 = 2.0  # dense int8 / dense bf16 tensor throughput (4.5 / 2.25 PFLOP/s nominal)
STEPS_PER_GRAPH = 10
TARGET_MIN_STEPS = 200   # steps of each target workload reported beside the headline


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=wl.HEADLINE, choices=sorted(wl.WORKLOADS))
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--sets", type=int, default=0,
                   help="rotating input sets (default: enough that a cycle touches 3x the L2); "
                        "1 keeps the device memory small, e.g. for a profiler capture")
    p.add_argument("--no-targets", action="store_true",
                   help="skip the FFN prefill and decode target workloads reported beside the headline")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the oracle baseline sample")
    p.add_argument("--out", default=None, help="also append the JSON line to this file")
    p.add_argument("--split", action="store_true",
                   help="shard W by output channel over the ranks (strong scaling) instead of "
                        "running a replica per rank")
    p.add_argument("--gather", action="store_true",
                   help="with --split: all-gather the Y shards every step (NCCL)")
    p.add_argument("--no-fp16-weights", action="store_true",
                   help="drop the fp16 weight: outlier-column weights come from CB * SCB / 127")
    p.add_argument("--quant", choices=["absmax", "zeropoint"], default="absmax",
                   help="absmax + outlier decomposition (LLM.int8()), or zeropoint on both sides")
    return p.parse_args()


# ------------------------------------------------------------------ peaks --

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def dram_traffic(kernel_key: str, source_files: list[str]):
    """Per-launch DRAM bytes from a committed ncu capture, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(kernel_key)
    if not d:
        return None
    h = hashlib.sha256()
    for s in source_files:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    if d.get("source_sha256") != h.hexdigest():
        return None
    return float(d["bytes_per_launch"]) * d.get("scale", 1.0)


# ----------------------------------------------------------------- clocks --

NVML_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    """Samples SM clock and clock-event reasons via NVML while running."""

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = None
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                ids = vis.split(",")
                if index < len(ids) and not ids[index].strip().isdigit():
                    uuid = ids[index].strip()
                elif index < len(ids):
                    index = int(ids[index])
            self.h = (pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid
                      else pynvml.nvmlDeviceGetHandleByIndex(index))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than fail the bench
            self.err = repr(e)

    def _sample(self):
        mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        try:
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append(mhz)
        self.reasons |= int(r)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        names = [n for bit, n in NVML_REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": names, "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------- CPU oracle --

def oracle_forward(w: wl.Workload, X, W, b, quant: str, keep_w: bool = True):
    """The oracle's forward of the chosen quantization, as a function of the row sample."""
    import oracle

    if quant == "zeropoint":
        CB, NDB, ZB, SB = oracle.zp_quantize_rows(W)
        return lambda rows: oracle.zp_forward(X, CB, NDB, ZB, SB, b, rows=rows)
    CB, SCB = oracle.prepare_weight(W)
    Wo = W if keep_w else None
    return lambda rows: oracle.forward(X, CB, SCB, Wo, w.threshold, b, rows=rows)


def cpu_oracle_sample(w: wl.Workload, target_s: float, X=None, W=None, quant: str = "absmax",
                      keep_w: bool = True):
    """Time the oracle forward on the first r rows of the workload (r sized to target_s)."""
    if X is None:
        X = wl.make_x(w)
    if W is None:
        W = wl.make_w(w)
    b = wl.make_bias(w)
    fwd = oracle_forward(w, X, W, b, quant, keep_w)   # weight conversion inside: offline, not timed
    probe = min(w.M, 8)
    t0 = time.perf_counter()
    fwd(np.arange(probe))
    per_row = (time.perf_counter() - t0) / probe          # upper bound: includes fixed costs
    rows = int(max(1, min(w.M, target_s / max(per_row, 1e-6))))
    t0 = time.perf_counter()
    fwd(np.arange(rows))
    dt = time.perf_counter() - t0
    if dt < 0.5 * target_s and rows < w.M:
        # the probe's fixed costs made the first sample short: size it again
        rows = int(max(1, min(w.M, rows * target_s / max(dt, 1e-6))))
        t0 = time.perf_counter()
        fwd(np.arange(rows))
        dt = time.perf_counter() - t0
    ops = 2.0 * rows * w.N * w.K
    what = ("outlier set over all rows, row quantize, int64-checked int8 GEMM, fp64 dequant + "
            "outlier product" if quant == "absmax" else
            "zeropoint row quantize, int64 int8 GEMM + zeropoint corrections, fp64 scale")
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": 1, "kind": "oracle",
            "sample": f"first {rows} of {w.M} rows x all {w.N} output channels ({what}); "
                      f"{dt:.2f} s on 1 host core",
            "host_cores": os.cpu_count(), "seconds": dt, "rows": rows}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    X, W = wl.make_x(w), wl.make_w(w)
    b = wl.make_bias(w)
    fwd = oracle_forward(w, X, W, b, args.quant, not getattr(args, "no_fp16_weights", False))
    t0 = time.perf_counter()
    fwd(np.arange(1))
    t_row = time.perf_counter() - t0
    budget = 150.0 / max(1, args.steps + args.warmup)      # whole run ~ 2.5 minutes
    rows = int(max(1, min(w.M, budget / max(t_row, 1e-6))))
    for _ in range(args.warmup):
        fwd(np.arange(rows))
    times = []
    for s in range(args.steps):
        r0 = (s * rows) % max(1, w.M - rows + 1)
        t0 = time.perf_counter()
        fwd(np.arange(r0, r0 + rows))
        times.append(time.perf_counter() - t0)
    total = sum(times)
    ops = 2.0 * rows * w.N * w.K * args.steps
    value = ops / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "n_outliers": w.n_outliers,
                   "threshold": w.threshold, "rows_per_step": rows, "quant": args.quant},
        "tokens_per_s": rows * args.steps / total,
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": 1, "kind": "oracle",
                         "sample": f"{rows} of {w.M} rows per step, all {w.N} output channels"},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(line, args.out)


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as tdist

    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return units_per_rank_step * steps * world / (max_ms * 1e-3)


def emit(line: dict, out: str | None):
    s = json.dumps(line)
    print(s, flush=True)
    if out:
        with open(out, "a") as f:
            f.write(s + "\n")


# -------------------------------------------------------------- GPU bench --

_W_CACHE: dict = {}


def weight_of(w: wl.Workload) -> np.ndarray:
    """W of a workload; workloads of one family (the decode sweep, the QKV sweep) share it."""
    key = (w.wid, w.N, w.K, w.sigma_w, w.seed)
    if key not in _W_CACHE:
        _W_CACHE.clear()
        _W_CACHE[key] = wl.make_w(w)
    return _W_CACHE[key]


def measure(args, w: wl.Workload, rank: int, world: int, local_rank: int, K_steps: int,
            warmup: int, with_e2e: bool) -> dict:
    """Time `K_steps` forwards of workload `w` (after `warmup` untimed ones) and each of its
    halves alone; with_e2e adds the pipelined host-buffer loop. Returns the measurements."""
    import torch

    from bit_quantized_matmul_int8_b200 import _lib

    dev = torch.device("cuda", local_rank)
    M, N, K = w.M, w.N, w.K
    N_full = N
    peaks = load_peaks()

    X = wl.make_x(w)
    W = weight_of(w)
    b = wl.make_bias(w)
    split = args.split and world > 1
    if split:
        # This rank's output channels; X is whole on every rank.
        from bit_quantized_matmul_int8_b200.shard import shard_rows

        n0, n1 = shard_rows(N, world, rank)
        if n1 <= n0:
            raise ValueError(f"--split: N={N} leaves rank {rank} of {world} no output channels")
        W = np.ascontiguousarray(W[n0:n1])
        b = np.ascontiguousarray(b[n0:n1]) if b is not None else None
        N = n1 - n0
    Xh = torch.from_numpy(X).pin_memory()
    Wd = torch.from_numpy(W).to(dev)
    keep_w = not args.no_fp16_weights and args.quant == "absmax"
    Wo = Wd if keep_w else None  # the fp16 weight the forward reads for the outlier columns
    bd = torch.from_numpy(b).to(dev) if b is not None else None
    zp = args.quant == "zeropoint"
    if zp:
        CB0, NDB, ZB, SB = _lib.int8lt_prepare_weight_zp(Wd)
    else:
        CB0, SCB = _lib.int8lt_prepare_weight(Wd)
    torch.cuda.synchronize()

    # The forward and its two halves, on one input set.
    def fwd(Xd, CB, Y, ws, st):
        if zp:
            _lib.int8lt_forward_zp(Xd, CB, NDB, ZB, SB, bd, Y, ws, st)
        else:
            _lib.int8lt_forward(Xd, CB, SCB, Wo, w.threshold, bd, Y, ws, st)

    def fwd_quantize(Xd, CB, ws, st):
        if zp:
            _lib.int8lt_forward_zp_quantize(Xd, N, ws, st)
        else:
            _lib.int8lt_forward_quantize(Xd, CB, SCB, Wo, w.threshold, ws, st)

    def fwd_matmul(CB, Y, ws, st):
        if zp:
            _lib.int8lt_forward_zp_matmul(M, K, CB, NDB, ZB, SB, bd, Y, ws, st)
        else:
            _lib.int8lt_forward_matmul(M, K, CB, SCB, Wo, bd, Y, ws, st)

    # Rotating input sets: X, CB, Y and workspace per set.
    ws_bytes = _lib.int8lt_workspace_size(M, N, K)
    touched = X.nbytes + M * K + (M * N * 2) + M * K + N * K  # X + CA + Y + CB(+CA write)
    R = int(min(16, max(3, math.ceil(3 * L2_BYTES / touched))))
    if getattr(args, "sets", 0) > 0:
        R = int(args.sets)
    Xs = [Xh.to(dev) for _ in range(R)]
    CBs = [CB0.clone() for _ in range(R)]
    Ys = [torch.empty((M, N), dtype=torch.float16, device=dev) for _ in range(R)]
    WSs = [_lib.workspace(M, N, K, dev) for _ in range(R)]
    del CB0
    stream = torch.cuda.current_stream()

    for s in range(max(3, warmup)):
        r = s % R
        fwd(Xs[r], CBs[r], Ys[r], WSs[r], stream)
    torch.cuda.synchronize()

    # The timed steps are replayed from CUDA graphs of up to STEPS_PER_GRAPH
    # whole steps each (quantize half, then matmul half, per step) with no
    # event nodes inside, so consecutive kernels overlap through programmatic
    # stream serialization as they do in a model's forward. (An event node
    # between two kernels stops that overlap and costs about 9 us per step
    # on the projection prefill.)
    decode = M <= 16
    cap_stream = torch.cuda.Stream(device=dev)

    def capture(s0, s1, quantize=True, matmul=True):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            cs = torch.cuda.current_stream()
            for s in range(s0, s1):
                r = s % R
                if quantize:
                    fwd_quantize(Xs[r], CBs[r], WSs[r], cs)
                if matmul:
                    fwd_matmul(CBs[r], Ys[r], WSs[r], cs)
        return g

    def graph_set(**kw):
        return [capture(s0, min(K_steps, s0 + STEPS_PER_GRAPH), **kw)
                for s0 in range(0, K_steps, STEPS_PER_GRAPH)]

    def replay_timed(gs):
        """Device ms of one pass over gs (after a warm-up pass), events on this stream."""
        for g in gs:
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for g in gs:
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    gather = split and args.gather
    if gather:
        from bit_quantized_matmul_int8_b200.shard import gather_shards

        # One graph per step; the all-gather of the Y shards runs between them.
        graphs = [capture(s0, s0 + 1) for s0 in range(K_steps)]
    else:
        graphs = graph_set()

    def replay_steps():
        for i, g in enumerate(graphs):
            g.replay()
            if gather:
                gather_shards(Ys[i % R], N_full)

    for _ in range(max(1, math.ceil(max(3, warmup) / K_steps))):
        replay_steps()
    torch.cuda.synchronize()

    dist = world > 1
    if dist:
        import torch.distributed as tdist
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    if dist:
        tdist.barrier()
    torch.cuda.synchronize()
    with sampler:
        t_start.record()
        replay_steps()
        t_end.record()
        torch.cuda.synchronize()
    if dist:
        tdist.barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    del graphs

    # Each half alone, over the same K steps and input rotation, replayed
    # back to back from graphs: the average launch duration of the quantize
    # kernel and of the matmul kernel (the roofline's dominant kernel).
    gq = graph_set(matmul=False)
    q_avg = replay_timed(gq) * 1e-3 / K_steps
    del gq
    gm = graph_set(quantize=False)
    m_sampler = ClockSampler(local_rank)
    with m_sampler:
        m_avg = replay_timed(gm) * 1e-3 / K_steps
    m_clocks = m_sampler.summary()
    del gm
    how = "each half alone over the same steps, back to back from graphs"
    if decode:
        # The decode GEMV's row blocks shared between warps are finished by
        # the last warp to arrive, counted on counters that the quantize pass
        # zeroes: replayed without it, the GEMV would skip those epilogues.
        # Its time is therefore the step's minus the quantize half's (alone).
        m_avg = max(elapsed_ms * 1e-3 / K_steps - q_avg, 0.0)
        how = ("quantize: alone over the same steps, back to back from graphs; matmul (GEMV): "
               "the step time minus the quantize half alone")
    for ws in WSs:
        st = _lib.int8lt_read_device_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {_lib.STATUS.get(st)} after the timed steps")

    ops = 2.0 * M * N * K                     # this rank's matmul per step
    if split:  # the ranks share one layer: the job does the whole layer per step
        value = 2.0 * M * N_full * K * K_steps / (elapsed_ms * 1e-3) / 1e12
        tokens_per_s = M * K_steps / (elapsed_ms * 1e-3)
    else:
        value = whole_job_rate(ops, K_steps, world, elapsed_ms) / 1e12
        tokens_per_s = whole_job_rate(M, K_steps, world, elapsed_ms)

    # Roofline of the dominant kernel: the matmul half is one launch (GEMM or GEMV).
    src = ["bit_quantized_matmul_int8_b200/csrc/gemm_tc.cu" if not decode
           else "bit_quantized_matmul_int8_b200/csrc/gemv.cu",
           "bit_quantized_matmul_int8_b200/csrc/int8lt_internal.cuh"]
    kname = (("gemm_i8_kernel" if not decode else "gemv_i8_kernel") + ("<zp>" if zp else "")
             + "@" + w.name)
    traffic = dram_traffic(kname, src)
    if not decode:
        # The kernel is timed alone: the burst peak. Where the power cap showed
        # while it was timed, the fraction of the sustained (power-capped)
        # figure is given beside it.
        peak = peaks["bf16_tflops"] * INT8_PER_BF16
        achieved = ops / m_avg / 1e12
        roof = {"bound": "tensor", "kernel": "gemm_i8_kernel", "achieved": achieved, "peak": peak,
                "unit": "TOPS", "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s"
                               f" x 2 (int8/bf16 nominal ratio)",
                "clocks_while_timed": m_clocks,
                "frac_of_sustained": (achieved / (peaks["bf16_tflops_sustained"] * INT8_PER_BF16)
                                      if "sw_power_cap" in m_clocks.get("reasons", []) else None),
                "algorithmic_units": f"2*M*N*K = {ops:.4g} int8 ops per launch"}
    else:
        if zp:  # CB + NDB/ZB/SB + CA + NDA/ZA/SA + Y
            alg_bytes = N * K + 12 * N + M * K + 12 * M + 2 * M * N
        else:
            n_out = w.n_outliers if math.isfinite(w.threshold) else 0
            alg_bytes = N * K + 4 * N + M * K + 4 * M + 2 * M * N + 2 * M * n_out + 2 * N * n_out
        achieved = alg_bytes / m_avg / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "kernel": "gemv_i8_kernel", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "traffic": traffic, "clocks_while_timed": m_clocks,
                "peak_source": f"{peaks['source']} HBM copy",
                "algorithmic_units": f"{alg_bytes} bytes per launch (CB + SCB + CA + SCA + Y + outliers)"
                                     if not zp else f"{alg_bytes} bytes per launch (CB + NDB/ZB/SB + CA"
                                                    f" + NDA/ZA/SA + Y)"}

    out = {
        "workload": w, "M": M, "N": N, "N_full": N_full, "K": K, "split": split, "gather": gather,
        "R": R, "touched": touched, "keep_w": keep_w, "zp": zp, "ws_bytes": ws_bytes,
        "steps": K_steps, "value": value, "ms_per_step": elapsed_ms / K_steps,
        "tokens_per_s": tokens_per_s, "clocks": sampler.summary(),
        "phases_ms": {"quantize": q_avg * 1e3, "matmul": m_avg * 1e3, "how": how},
        "roofline": roof, "X": X, "W": W,
    }
    if not with_e2e:
        return out

    # End to end through the public API, as a serving loop runs it: every step
    # copies its X in from pinned host memory, runs int8lt_forward and copies Y
    # out to pinned host memory. Copies in, compute and copies out go on three
    # streams over two buffer slots, so a step's copies overlap the neighbouring
    # steps' work (PCIe carries both directions at once).
    slots = 2
    layer_ws = WSs[0]
    Xds = [torch.empty_like(Xs[0]) for _ in range(slots)]
    Yds = [torch.empty_like(Ys[0]) for _ in range(slots)]
    Yhs = [torch.empty((M, N), dtype=torch.float16).pin_memory() for _ in range(slots)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_done = [torch.cuda.Event() for _ in range(slots)]
    comp_done = [torch.cuda.Event() for _ in range(slots)]
    out_done = [torch.cuda.Event() for _ in range(slots)]

    def e2e_steps(n):
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for i in range(n):
            k = i % slots
            if i >= slots:
                s_in.wait_event(comp_done[k])      # the forward two steps back read Xds[k]
            with torch.cuda.stream(s_in):
                Xds[k].copy_(Xh, non_blocking=True)
                in_done[k].record(s_in)
            stream.wait_event(in_done[k])
            if i >= slots:
                stream.wait_event(out_done[k])     # Yds[k] has been copied out
            fwd(Xds[k], CBs[0], Yds[k], layer_ws, stream)
            comp_done[k].record(stream)
            s_out.wait_event(comp_done[k])
            with torch.cuda.stream(s_out):
                Yhs[k].copy_(Yds[k], non_blocking=True)
                out_done[k].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    e2e_steps(3)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = min(K_steps, 100)
    if dist:
        tdist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    e2e_steps(n_e2e)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_ops = 2.0 * M * N_full * K / world if split else ops  # per rank, whole job = x world
    out["e2e"] = {"value": whole_job_rate(e2e_ops, n_e2e, world, e2e_ms) / 1e12, "unit": "TOPS",
                  "h2d_bytes_per_step": int(Xh.numel() * 2), "d2h_bytes_per_step": int(Yhs[0].numel() * 2),
                  "pipeline": "copy-in / forward / copy-out on three streams, two buffer slots",
                  "steps": n_e2e,
                  "tokens_per_s": whole_job_rate(M, n_e2e, world, e2e_ms) / (world if split else 1)}
    return out


def clock_scaled(ms: float, clocks: dict) -> dict:
    """The step time with the SM clock it ran at: ms x median MHz, and the time it
    would take at the maximum clock if it scaled with the clock alone."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if not mhz or not mx:
        return {}
    return {"ms_x_sm_mhz": ms * mhz, "ms_at_max_clock": ms * mhz / mx}


def target_summary(r: dict) -> dict:
    """The figures of one target workload, for the JSON line's `targets` object."""
    roof = r["roofline"]
    d = {"ms_per_step": r["ms_per_step"], "steps": r["steps"], "value": r["value"], "unit": "TOPS",
         "tokens_per_s": r["tokens_per_s"], "phases_ms": r["phases_ms"],
         "dominant_kernel": {k: roof[k] for k in ("kernel", "bound", "achieved", "peak", "unit", "frac",
                                                  "frac_of_sustained") if k in roof},
         "clocks": r["clocks"], "clocks_while_timed": roof["clocks_while_timed"]}
    d.update(clock_scaled(r["ms_per_step"], r["clocks"]))
    return d


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch

    from bit_quantized_matmul_int8_b200 import _lib, build

    build.build()
    torch.cuda.set_device(local_rank)
    w = wl.WORKLOADS[args.workload]
    r = measure(args, w, rank, world, local_rank, args.steps, args.warmup, with_e2e=True)
    M, N, N_full, K = r["M"], r["N"], r["N_full"], r["K"]
    X, W = r.pop("X"), r.pop("W")
    zp, keep_w, split = r["zp"], r["keep_w"], r["split"]

    # The other target shapes, each timed the same way over its own steps (at
    # least TARGET_MIN_STEPS, so that every timed region spans a few clock samples).
    targets = {}
    if not args.no_targets and not split:
        for name in wl.TARGETS:
            if name == w.name:
                continue
            torch.cuda.empty_cache()
            t = measure(args, wl.WORKLOADS[name], rank, world, local_rank,
                        max(args.steps, TARGET_MIN_STEPS), args.warmup, with_e2e=False)
            targets[name] = target_summary(t)
            del t
    torch.cuda.empty_cache()

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": r["value"], "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
        "scaling": "strong" if split else "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": w.name, "M": M, "K": K, "N": N_full, "n_outliers": w.n_outliers,
                   "threshold": w.threshold, "x": "N(0,1) fp16 + planted outlier columns",
                   "w": f"N(0,{w.sigma_w}) fp16", "l2": f"{r['R']} rotating input sets "
                   f"({r['R'] * r['touched'] / 2**20:.0f} MiB touched per cycle) > 126 MB L2",
                   "parallelism": (f"N split x{world} ({N} channels per rank"
                                   + (", Y all-gathered" if r["gather"] else "") + ")") if split
                   else f"replicas x{world}", "quant": args.quant,
                   "cuda_graphs": f"up to {STEPS_PER_GRAPH} whole steps per graph, no event nodes inside"},
        "tokens_per_s": r["tokens_per_s"],
        "memory": {"layer_bytes": _lib.int8lt_weight_bytes(N, K) + (12 * N if zp else 4 * N)
                   + (2 * N * K if keep_w else 0),
                   "fp16_layer_bytes": 2 * N * K, "fp16_weight_kept": keep_w,
                   "workspace_bytes": r["ws_bytes"]},
        "phases_ms": r["phases_ms"],
        "roofline": r["roofline"],
        "e2e": r["e2e"],
        "gpu_launches": args.steps * 2,  # the quantize kernel + the GEMM or GEMV, per step
        "clocks": r["clocks"],
    }
    line.update({k: v for k, v in clock_scaled(r["ms_per_step"], r["clocks"]).items()})
    if targets:
        line["targets"] = targets
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_oracle_sample(w, args.cpu_seconds, X, W, args.quant, keep_w)
    elif not args.no_cpu_baseline:
        line["cpu_baseline"] = None
    emit(line, args.out)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist

        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as tdist

            tdist.destroy_process_group()


if __name__ == "__main__":
    main()
