#!/usr/bin/env python
"""Benchmark of the VQ dequantize-and-multiply hot path on B200.

One step = the whole hot path of the dense MLP trio at d2/K256 with k-means codebooks
(gate and up [17408][5120], down [5120][17408]):
  * decode: one token through the trio (three GEMV launches, fp16 activations, fp32
    outputs);
  * prefill: 2048 bf16 tokens through the trio (three tensor-core GEMM launches, bf16
    outputs; the bf16 activations are converted to fp16 inside vq_gemm).
Three copies of the trio (3 x 142 MB) rotate, so no step finds its weights in the 126 MB
L2.  The MoE layers (256 experts top-8 with mixed tiers; 512 experts top-10) are timed
as extra legs of the same run, with L2 flushed between iterations.

`value` is the decode GEMV's effective HBM bandwidth (algorithmic bytes: packed codes +
scales + codebook + x + y, over the decode launches' device time); `prefill` holds the
prefill TFLOP/s; `moe` the MoE layers' tokens/s.  Inputs are synthetic and seeded
(workloads package).

`python bench.py [--gpus N] [--steps K] [--warmup W]` prints one JSON line.  With N > 1
(torchrun) every rank runs an independent replica (the path has no exchange step) and
the line reports whole-job throughput over the max-over-ranks device time.
`--impl reference` times the CPU oracle on the host cores instead (a bounded sample of
the same workload per step).
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

GEMV_TRAFFIC_BYTES = 47_408_000.0
METRIC = "VQ GEMV effective HBM GB/s (% of peak); prefill TFLOP/s; MoE layer tokens/s"
PREFILL_TOKENS = 2048
COPIES = 3
L2_FLUSH_BYTES = 256 << 20


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


# ----------------------------------------------------------------------------- algorithmic sizes

def weight_bytes(data, experts=1):
    """Packed codes + fp16 scales (+ one codebook) of a tensor."""
    rb = ((data.cols // data.d + 31) // 32) * 4 * data.bits
    return experts * (data.rows * rb + data.rows * (data.cols // 64) * 2) + (1 << data.bits) * data.d * 2


def gemv_bytes(data, x_el=2, y_el=4, batch=1):
    """Algorithmic bytes of one GEMV: packed codes + scales + codebook + x + y."""
    return weight_bytes(data) + batch * data.cols * x_el + batch * data.rows * y_el


def gemm_flops(data, M):
    return 2.0 * M * data.rows * data.cols


def _dev_bits(a, dev, dtype):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(dtype)


# ----------------------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import torch

    import vq_dequant_matmul_b200 as vq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pk = peaks()
    stream = torch.cuda.current_stream()

    trio = wl.c2_mlp_tensors(device=str(dev))
    mats = [[vq.VQMatrix.from_data(t, device=dev) for t in trio]]
    for _ in range(COPIES - 1):
        mats.append([vq.VQMatrix(m.codebook.clone(), m.codes.clone(), m.scales.clone(), m.rows, m.cols,
                                 m.d, m.bits) for m in mats[0]])
    # decode inputs / outputs
    xd = [_dev_bits(wl.activations(1, t.cols, wl.BASE_SEED + 10 + i, wl.F16), dev, torch.float16)
          for i, t in enumerate(trio)]
    yd = [torch.empty((1, t.rows), dtype=torch.float32, device=dev) for t in trio]
    # prefill inputs / outputs (bf16 activations and outputs)
    M = PREFILL_TOKENS
    xp = [_dev_bits(wl.activations(M, t.cols, wl.BASE_SEED + 20 + i, wl.BF16), dev, torch.bfloat16)
          for i, t in enumerate(trio)]
    yp = [torch.empty((M, t.rows), dtype=torch.bfloat16, device=dev) for t in trio]
    ws_bytes = max(vq.vq_gemm_workspace_size(mats[0][i], torch.bfloat16, M) for i in range(3))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    dec_bytes = [gemv_bytes(t) for t in trio]
    pre_flops = [gemm_flops(t, M) for t in trio]

    def step(c, ev=None):
        # the three decode GEMVs, then the three prefill GEMMs, each block back to back
        # (consecutive launches overlap through programmatic dependent launch, so a block
        # is timed as a whole)
        if ev is not None:
            ev[0][0].record(stream)
        for i in range(3):
            vq.vq_gemv(mats[c][i], xd[i], yd[i])
        if ev is not None:
            ev[0][1].record(stream)
            ev[1][0].record(stream)
        for i in range(3):
            vq.vq_gemm(mats[c][i], xp[i], yp[i], ws)
        if ev is not None:
            ev[1][1].record(stream)

    for s in range(args.warmup):
        step(s % COPIES)
    torch.cuda.synchronize()

    K = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(2)] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        start.record(stream)
        for s in range(K):
            step(s % COPIES, evs[s])
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(start.elapsed_time(stop), world)
    blk_ms = [sum(evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(K)) / K for i in range(2)]
    dec_ms = max_over_ranks(blk_ms[0], world)
    pre_ms = max_over_ranks(blk_ms[1], world)
    value = job_throughput(sum(dec_bytes), dec_ms, world) / 1e9
    prefill_tflops = job_throughput(sum(pre_flops), pre_ms, world) / 1e12

    # context (not the timed region): each projection timed alone, one launch between events
    iso = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(6)]
    iso_ms = [0.0] * 6
    NI = 10
    for s in range(NI):
        c = s % COPIES
        for i in range(3):
            iso[i][0].record(stream)
            vq.vq_gemv(mats[c][i], xd[i], yd[i])
            iso[i][1].record(stream)
        for i in range(3):
            iso[3 + i][0].record(stream)
            vq.vq_gemm(mats[c][i], xp[i], yp[i], ws)
            iso[3 + i][1].record(stream)
        torch.cuda.synchronize()
        for i in range(6):
            iso_ms[i] += iso[i][0].elapsed_time(iso[i][1]) / NI

    gemv_gbs = sum(dec_bytes) / (blk_ms[0] * 1e-3) / 1e9
    roofline = {"kernel": "gemv_mma_kernel<2,8,1,1,1> (mma.sync, 16-row A-operand blocks, TMA stages, 2-4 CTA clusters)",
                "bound": "hbm", "achieved": round(gemv_gbs, 1),
                "peak": pk["hbm"], "unit": "GB/s", "frac": round(gemv_gbs / pk["hbm"], 4),
                "traffic": args.traffic or None, "peak_source": pk["source"] + " (burst copy)",
                "launch_ms": round(blk_ms[0] / 3, 5),
                "per_projection_isolated_gbs": [round(dec_bytes[i] / (iso_ms[i] * 1e-3) / 1e9, 1) for i in range(3)],
                "frac_of_nominal_8tbs": round(gemv_gbs / 8000.0, 4)}
    gemm_tf = sum(pre_flops) / (blk_ms[1] * 1e-3) / 1e12
    prefill = {"value": round(prefill_tflops, 1), "unit": "TFLOP/s", "ms": round(pre_ms, 4),
               "tokens": M, "flops": sum(pre_flops),
               "roofline": {"kernel": "vq_gemm_kernel<256|192 tokens> (tcgen05, fp16 A tiles in tensor memory, TMA code blocks)", "bound": "tensor",
                            "achieved": round(gemm_tf, 1), "peak": pk["bf16_sus"], "unit": "TFLOP/s",
                            "frac": round(gemm_tf / pk["bf16_sus"], 4),
                            "frac_of_burst_peak": round(gemm_tf / pk["bf16"], 4),
                            "peak_source": pk["source"] + " (sustained bf16 cuBLAS; fp16 has the same rate)",
                            "traffic": None,
                            "per_projection_isolated_tflops": [round(pre_flops[i] / (iso_ms[3 + i] * 1e-3) / 1e12, 1)
                                                               for i in range(3)]}}

    # end to end through the C ABI: pinned host inputs -> device, step, outputs -> pinned host
    xh = [x.cpu().pin_memory() for x in xd + xp]
    yh = [torch.empty_like(y, device="cpu").pin_memory() for y in yd + yp]
    xdev, ydev = xd + xp, yd + yp
    h2d = sum(x.numel() * x.element_size() for x in xh)
    d2h = sum(y.numel() * y.element_size() for y in yh)
    K2 = max(3, min(K, args.e2e_steps))

    def e2e_step(c):
        for i in range(6):
            xdev[i].copy_(xh[i], non_blocking=True)
        step(c)
        for i in range(6):
            yh[i].copy_(ydev[i], non_blocking=True)

    for s in range(3):
        e2e_step(s % COPIES)
    torch.cuda.synchronize()
    barrier(world)
    start.record(stream)
    for s in range(K2):
        e2e_step(s % COPIES)
    stop.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(start.elapsed_time(stop), world) / K2
    e2e = {"value": round(sum(dec_bytes) * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
           "steps": K2,
           "note": "decode bytes over the whole end-to-end step (decode + 2048-token prefill + copies)"}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(total_ms / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": "dense MLP trio d2/K256 k-means codebooks (gate/up 17408x5120, down "
                               "5120x17408): batch-1 fp16 decode + 2048-token bf16 prefill per step",
                   "decode_bytes_per_step": sum(dec_bytes), "prefill_flops_per_step": sum(pre_flops),
                   "l2": f"{COPIES} weight copies rotated (3 x 142 MB > 126 MB L2)",
                   "parallelism": f"replicas{world}"},
        "roofline": roofline, "prefill": prefill, "e2e": e2e,
        "clocks": clk.summary(),
    }
    # timed region: per step 3 GEMV launches + 3 x (bf16->fp16 conversion + GEMM)
    line["gpu_launches"] = 9 * K
    if not args.no_moe:
        line["moe"] = moe_legs(args, vq, dev, pk, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(trio, args.cpu_rows)
    return line


def moe_legs(args, vq, dev, pk, world):
    """Routed MoE layers: tokens/s per (layer, T), L2 flushed between timed iterations."""
    import torch

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    out = {}
    for name, builder, Ts in (("c4_256x_top8_mixed", wl.c4_moe, (1, 16, 512)),
                              ("c5_512x_top10_d4k256", wl.c5_moe_large, (1, 1024))):
        mw = builder()
        G, U, D = (vq.VQMatrix.from_data(t, device=dev) for t in (mw.gate, mw.up, mw.down))
        per_expert = sum(weight_bytes(t) - (1 << t.bits) * t.d * 2 for t in (mw.gate, mw.up, mw.down))
        cbs = sum((1 << t.bits) * t.d * 2 for t in (mw.gate, mw.up, mw.down))
        for T in Ts:
            nrep = 8
            inputs = []
            for r in range(nrep):
                x, ids, w = wl.moe_inputs(mw, T, seed=wl.BASE_SEED + 300 + 17 * r + T)
                inputs.append((_dev_bits(x, dev, torch.float16), torch.from_numpy(ids).to(dev),
                               torch.from_numpy(w).to(dev), len(np.unique(ids))))
            y = torch.empty((T, mw.hidden), dtype=torch.float32, device=dev)
            ws = torch.empty(vq.vq_moe_workspace_size(T, mw.topk, mw.E, mw.hidden, mw.inter),
                             dtype=torch.uint8, device=dev)
            for r in range(3):
                xdv, idd, wd, _ = inputs[r % nrep]
                vq.vq_moe_grouped(G, U, D, xdv, idd, wd, y, ws)
            torch.cuda.synchronize()
            iters = args.moe_iters
            times, nbytes = [], []
            for it in range(iters):
                xdv, idd, wd, ne = inputs[it % nrep]
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                vq.vq_moe_grouped(G, U, D, xdv, idd, wd, y, ws)
                e1.record(stream)
                times.append((e0, e1))
                nbytes.append(ne * per_expert + cbs + T * mw.hidden * 2 * 2)
            torch.cuda.synchronize()
            ms = [a.elapsed_time(b) for a, b in times]
            mean_ms = max_over_ranks(sum(ms) / len(ms), world)
            gbs = sum(nbytes) / len(nbytes) / (mean_ms * 1e-3) / 1e9
            out[f"{name}_T{T}"] = {"tokens_per_s": round(T * world / (mean_ms * 1e-3), 1), "ms": round(mean_ms, 4),
                                   "effective_gbs": round(gbs, 1), "hbm_frac": round(gbs / pk["hbm"], 4),
                                   "path": "grouped tcgen05 GEMM" if T * mw.topk / min(mw.E, T * mw.topk) >= 4
                                   else "grouped GEMV", "iters": iters, "l2": "flushed between iterations"}
            out[f"{name}_T{T}"]["gpu_launches"] = iters * (6 if out[f"{name}_T{T}"]["path"].startswith("grouped tc")
                                                            else 4)
            del ws, y
        del G, U, D, mw
        torch.cuda.empty_cache()
    return out


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v, world):
    """The largest value over the ranks (device times: the job takes as long as the slowest)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, max_ms, world):
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / (max_ms * 1e-3)


# ----------------------------------------------------------------------------- oracle arm

def _oracle_sample(trio, rows):
    import oracle

    subs = []
    for i, t in enumerate(trio):
        sub = wl.VQTensorData(min(rows, t.rows), t.cols, t.d, t.bits, t.codebook,
                              t.codes[:, :rows], t.scales[:, :rows])
        subs.append((oracle.Tensor(sub), gemv_bytes(sub), wl.activations(1, t.cols, wl.BASE_SEED + 10 + i, wl.F16)))
    return subs


def cpu_baseline(trio, rows):
    """The oracle (as it stands) on a bounded sample: the first `rows` rows of each
    projection of the decode step, compute only.  Same unit (effective GB/s)."""
    import oracle

    subs = _oracle_sample(trio, rows)
    t1 = time.perf_counter()
    for ot, _, x in subs:
        ot.linear(x, wl.F16)
    dt = time.perf_counter() - t1
    nbytes = sum(b for _, b, _ in subs)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {rows} rows of each of gate/up/down, batch-1 decode ({nbytes} algorithmic bytes), "
                      f"{dt:.2f} s"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: every step is the bounded decode sample."""
    if rank != 0:
        return None
    import oracle

    trio = wl.c2_mlp_tensors(device="cuda" if _cuda() else "cpu")
    subs = _oracle_sample(trio, args.cpu_rows)
    nbytes = sum(b for _, b, _ in subs)
    for _ in range(args.warmup):
        for ot, _, x in subs:
            ot.linear(x, wl.F16)
    t1 = time.perf_counter()
    for _ in range(args.steps):
        for ot, _, x in subs:
            ot.linear(x, wl.F16)
    dt = time.perf_counter() - t1
    v = nbytes * args.steps / dt / 1e9
    sample = f"first {args.cpu_rows} rows of each of gate/up/down, batch-1 decode ({nbytes} bytes per step)"
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
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=2048)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--moe-iters", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-moe", action="store_true")
    # dram__bytes_read.sum + dram__bytes_write.sum per launch of the decode GEMV, mean of the
    # gate / up / down launches of one ncu capture of this kernel version
    # (profiles/gemv_mma_c2_decode.md); pass 0 to report null
    ap.add_argument("--traffic", type=float, default=GEMV_TRAFFIC_BYTES,
                    help="dram bytes per launch of the decode GEMV from an ncu capture (0: null)")
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
