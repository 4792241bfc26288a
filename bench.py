#!/usr/bin/env python
"""Benchmark of the VQ dequantize-and-multiply hot path on B200.

Workload (one "step"): the dense MLP trio at d2/K256 with k-means codebooks (gate and
up [17408][5120], down [5120][17408]): one decode token through the trio (three GEMV
launches, fp16 activations, fp32 outputs) and one 2048-token bf16 prefill through the
trio (three tensor-core GEMM launches).  Inputs are synthetic and seeded (workloads
package); three copies of the trio (3 x 142 MB) are rotated so that no step finds its
weights in the 126 MB L2.

`python bench.py [--gpus N] [--steps K] [--warmup W]` prints one JSON line.  With N > 1
(torchrun) every rank runs an independent replica (the path has no exchange step) and the
line reports the whole-job throughput over the max-over-ranks device time.
`--impl reference` times the CPU oracle on the host cores instead (a bounded sample of the
same workload per step).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "VQ GEMV effective HBM GB/s (% of peak); prefill TFLOP/s; MoE layer tokens/s"
PREFILL_TOKENS = 2048
COPIES = 3


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sus": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.15)
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- workload bytes

def gemv_bytes(data, x_el=2, y_el=4, batch=1):
    """Algorithmic bytes of one GEMV: packed codes + scales + codebook + x + y."""
    rb = ((data.cols // data.d + 31) // 32) * 4 * data.bits
    return (data.rows * rb + data.rows * (data.cols // 64) * 2 + (1 << data.bits) * data.d * 2
            + batch * data.cols * x_el + batch * data.rows * y_el)


# ----------------------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import torch

    import vq_dequant_matmul_b200 as vq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pk = peaks()

    trio = wl.c2_mlp_tensors(device=str(dev))
    mats = [[vq.VQMatrix.from_data(t, device=dev) for t in trio]]
    for _ in range(COPIES - 1):
        mats.append([vq.VQMatrix(m.codebook.clone(), m.codes.clone(), m.scales.clone(), m.rows, m.cols,
                                 m.d, m.bits) for m in mats[0]])
    xd = [torch.from_numpy(wl.activations(1, t.cols, wl.BASE_SEED + 10 + i, wl.F16).view(np.int16))
          .to(dev).view(torch.float16) for i, t in enumerate(trio)]
    yd = [torch.empty((1, t.rows), dtype=torch.float32, device=dev) for t in trio]
    dec_bytes = [gemv_bytes(t) for t in trio]
    step_bytes = sum(dec_bytes)
    stream = torch.cuda.current_stream()

    def decode(c, ev=None):
        for i in range(3):
            if ev is not None:
                ev[i][0].record(stream)
            vq.vq_gemv(mats[c][i], xd[i], yd[i])
            if ev is not None:
                ev[i][1].record(stream)

    # warm-up
    for s in range(args.warmup):
        decode(s % COPIES)
    torch.cuda.synchronize()

    # timed region: K steps, per-launch events on the launching stream
    K = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        start.record(stream)
        for s in range(K):
            decode(s % COPIES, evs[s])
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = start.elapsed_time(stop)
    kern_ms = [sum(evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(K)) for i in range(3)]
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / K
    value = step_bytes * K * world / (total_ms * 1e-3) / 1e9

    gemv_ms = sum(kern_ms) / (3 * K)
    gemv_gbs = step_bytes / 3 / (gemv_ms * 1e-3) / 1e9
    roofline = {"kernel": "gemv_b1_kernel<2,8,half>", "bound": "hbm", "achieved": round(gemv_gbs, 1),
                "peak": pk["hbm"], "unit": "GB/s", "frac": round(gemv_gbs / pk["hbm"], 4),
                "traffic": args.traffic, "peak_source": pk["source"],
                "per_projection_gbs": [round(dec_bytes[i] / (kern_ms[i] / K * 1e-3) / 1e9, 1) for i in range(3)]}

    # end to end through the C ABI: pinned host x -> device, GEMVs, device y -> pinned host
    xh = [x.cpu().pin_memory() for x in xd]
    yh = [torch.empty_like(y, device="cpu").pin_memory() for y in yd]
    h2d = sum(x.numel() * x.element_size() for x in xh)
    d2h = sum(y.numel() * y.element_size() for y in yh)
    for s in range(args.warmup):
        for i in range(3):
            xd[i].copy_(xh[i], non_blocking=True)
        decode(s % COPIES)
        for i in range(3):
            yh[i].copy_(yd[i], non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    start.record(stream)
    for s in range(K):
        for i in range(3):
            xd[i].copy_(xh[i], non_blocking=True)
        decode(s % COPIES)
        for i in range(3):
            yh[i].copy_(yd[i], non_blocking=True)
    stop.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(start.elapsed_time(stop), world)
    e2e = {"value": round(step_bytes * K * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / K, 5)}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": "dense MLP trio d2/K256 (gate/up 17408x5120, down 5120x17408), "
                               "batch-1 decode through the trio",
                   "weights_bytes_per_step": step_bytes, "l2": f"{COPIES} weight copies rotated (> L2)",
                   "parallelism": f"replicas{world}"},
        "frac_of_nominal_8tbs": round(value / 8000.0, 4),
        "roofline": roofline, "e2e": e2e, "gpu_launches": 3 * K,
    }
    clocks = clk.summary()
    line["clocks"] = clocks
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_decode(trio, args.cpu_rows)
    return line


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- oracle arm

def cpu_baseline_decode(trio, rows_per_proj):
    """The oracle (as it stands) on a bounded sample: the first `rows_per_proj` rows of
    each projection of the decode step, compute only (packing is input preparation).
    Reported in the same unit (effective GB/s)."""
    import oracle

    t_all, nbytes = 0.0, 0
    for i, t in enumerate(trio):
        sub = wl.VQTensorData(min(rows_per_proj, t.rows), t.cols, t.d, t.bits, t.codebook,
                              t.codes[:, :rows_per_proj], t.scales[:, :rows_per_proj])
        ot = oracle.Tensor(sub)
        x = wl.activations(1, t.cols, wl.BASE_SEED + 10 + i, wl.F16)
        t1 = time.perf_counter()
        ot.linear(x, wl.F16)
        t_all += time.perf_counter() - t1
        nbytes += gemv_bytes(sub)
    return {"value": round(nbytes / t_all / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"first {rows_per_proj} rows of each of gate/up/down, batch-1 decode "
                      f"({nbytes} algorithmic bytes), {t_all:.2f} s"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: every step is the bounded decode sample."""
    if rank != 0:
        return None
    import oracle

    trio = wl.c2_mlp_tensors(device="cuda" if _cuda() else "cpu")
    rows = args.cpu_rows
    subs, xs = [], []
    for i, t in enumerate(trio):
        sub = wl.VQTensorData(min(rows, t.rows), t.cols, t.d, t.bits, t.codebook,
                              t.codes[:, :rows], t.scales[:, :rows])
        subs.append((oracle.Tensor(sub), gemv_bytes(sub)))
        xs.append(wl.activations(1, t.cols, wl.BASE_SEED + 10 + i, wl.F16))
    nbytes = sum(b for _, b in subs)
    for _ in range(args.warmup):
        for (ot, _), x in zip(subs, xs):
            ot.linear(x, wl.F16)
    t1 = time.perf_counter()
    for _ in range(args.steps):
        for (ot, _), x in zip(subs, xs):
            ot.linear(x, wl.F16)
    dt = time.perf_counter() - t1
    v = nbytes * args.steps / dt / 1e9
    sample = f"first {rows} rows of each of gate/up/down, batch-1 decode ({nbytes} bytes per step)"
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "dense MLP trio d2/K256, batch-1 decode (oracle sample)"},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def _cuda():
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=2048)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_ours(args, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
