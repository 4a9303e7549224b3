#!/usr/bin/env python
"""Benchmark of the SSA hot path on B200.

Step = one SSA prefill (MLA-absorbed, one sequence of 32,768 tokens, 64 query
heads sharing a 576-wide latent KV whose first 512 columns are V, scale
1/sqrt(192), b=128 s=1 l=7) over inputs already resident in HBM; the metric is
algorithmic TFLOP/s (2*(576+512) FLOP per visible (query, key) pair per head).
The same line carries the roofline of the prefill kernel, the fp64 CPU oracle
timed on a bounded sample of the same workload, an end-to-end figure through
the public API with host buffers, and (when available) the decode kernel's
achieved HBM bandwidth.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch under torch.distributed.run; every rank runs its own replica
of the workload (independent problems, no collective in the data path) and the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

B, S, LW = 128, 1, 7
WORKLOAD = synth.WORKLOADS[2]
SEQLEN = WORKLOAD["seqlen"]
H, DQK, DV = WORKLOAD["n_heads"], WORKLOAD["d_qk"], WORKLOAD["d_v"]
SCALE = WORKLOAD["scale"]
METRIC = "SSA prefill TFLOP/s & decode GB/s at 32K-1M ctx, % of B200 roofline"
UNIT = "TFLOP/s"


def visible_pairs(L, b=B, s=S, l=LW):
    """Sum over queries of the number of visible keys (closed form per block)."""
    total = 0
    for j in range((L + b - 1) // b):
        lo, hi = j * b, min(L, (j + 1) * b)
        n = hi - lo
        if j < s + l - 1:
            total += (lo + 1 + hi) * n // 2
        else:
            total += n * (s * b + (l - 1) * b + 1) + (n * (n - 1)) // 2
    return total


def prefill_flops(L=SEQLEN):
    return 2.0 * (DQK + DV) * H * visible_pairs(L)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_streaming_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_counters.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(1.0)  # let the sampler start before the timed region
        return self

    def mark(self, which):
        """Wall-clock bounds of the timed region; samples outside are dropped."""
        setattr(self, which, time.time())

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        import datetime
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0, t1 = getattr(self, "t0", None), getattr(self, "t1", None)
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if t0 is not None and not (t0 - 0.05 <= ts <= t1 + 0.05):
                    continue
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- oracle (CPU) leg

def oracle_sample(n_rows_target_s=15.0, rank_seed=0):
    """Time the fp64 oracle on a bounded sample of the prefill workload: query rows
    spread over the sequence (all 64 heads of each). Returns (TFLOP/s, desc, cores)."""
    import oracle
    oracle.build()
    g = synth.rng(synth.workload_seed(2))
    L = SEQLEN
    # the latent KV in full (37.7 MB); Q only for the sampled rows
    lat = synth.normal_bits(g, (L, 1, DQK))
    vlat = np.ascontiguousarray(lat[:, :, :DV])
    cu = synth.cu_seqlens([L])
    q = np.zeros((L, H, DQK), np.uint16)
    rs = np.random.default_rng(12345 + rank_seed)

    def run(n):
        rows = np.sort(rs.choice(np.arange(1024, L), size=n, replace=False))
        q[rows] = synth.normal_bits(rs, (n, H, DQK))
        t0 = time.perf_counter()
        oracle.forward(q, lat, vlat, cu, H, 1, B, S, LW, SCALE, rows=rows)
        dt = time.perf_counter() - t0
        pairs = sum(min(r + 1, S * B + (LW - 1) * B + (r % B) + 1) for r in rows)
        return dt, 2.0 * (DQK + DV) * H * pairs, rows

    dt, fl, _ = run(4)
    n = int(max(4, min(4096, 4 * n_rows_target_s / max(dt, 1e-3))))
    dt, fl, rows = run(n)
    cores = len(os.sched_getaffinity(0))
    desc = (f"{n} query rows (all {H} heads) sampled uniformly from positions 1024..{L - 1} of the "
            f"L={L} absorbed prefill; fp64 oracle, {cores} OpenMP threads, {dt:.1f} s")
    return fl / dt / 1e12, desc, cores, dt


def run_reference(args, rank, world):
    if rank != 0:
        return
    per = []
    desc = cores = None
    for i in range(args.warmup + args.steps):
        v, desc, cores, dt = oracle_sample(n_rows_target_s=8.0, rank_seed=i)
        if i >= args.warmup:
            per.append((v, dt))
    value = statistics.mean(v for v, _ in per)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * statistics.mean(dt for _, dt in per), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD["name"], "seq_len": SEQLEN, "n_heads": H, "d_qk": DQK, "d_v": DV,
                   "block": [B, S, LW]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU leg

def make_inputs(device, seed_offset=0):
    import torch
    seed = synth.workload_seed(2) * 1000 + seed_offset
    q = synth.torch_normal_bf16((SEQLEN, H, DQK), seed, device)
    lat = synth.torch_normal_bf16((SEQLEN, 1, DQK), seed + 1, device)
    cu = torch.tensor([0, SEQLEN], dtype=torch.int32, device=device)
    return q, lat, cu


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import block_sparse_streaming_b200 as bss

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    bss.lib()
    params = bss.Params(SCALE, B, S, LW)
    q, lat, cu = make_inputs(device, seed_offset=rank)
    v = lat[:, :, :DV]
    out = torch.empty((SEQLEN, H, DV), dtype=torch.bfloat16, device=device)
    lse = torch.empty((SEQLEN, H), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step():
        bss.loza_ssa_prefill(q, lat, v, cu, SEQLEN, params, out=out, lse=lse, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches0 = bss.launch_count()
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        clk.mark("t0")
        t_all0.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize()
        clk.mark("t1")
        if world > 1:
            dist.barrier()
    launches = bss.launch_count() - launches0
    total_ms = t_all0.elapsed_time(t_all1)
    per_launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    status = bss.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    t = torch.tensor([total_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    flops = prefill_flops()
    value = world * args.steps * flops / (total_ms / 1000.0) / 1e12

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(bss, params, device, stream, steps=max(1, min(args.steps, 3)))

    peaks, peak_kind = measured_peaks()
    avg_launch_ms = statistics.mean(per_launch_ms)
    achieved = flops / (avg_launch_ms / 1000.0) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = profiled_traffic("ssa_prefill_kernel<576,256,5>")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "peak_kind": f"{peak_kind} bf16 dense burst (MEASURED_PEAKS.json bf16_tflops)",
                "kernel": "ssa_prefill_kernel<576,256,5>",
                "algorithmic_flop_per_launch": flops}

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v_cpu, desc, cores, _ = oracle_sample()
            cpu = {"value": v_cpu, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD["name"], "batch": 1, "seq_len": SEQLEN, "n_heads": H,
                       "kv": "shared latent 576 (V = first 512)", "d_qk": DQK, "d_v": DV,
                       "block": [B, S, LW], "parallelism": f"replica x{world}",
                       "l2": "inputs larger than L2 (Q is 2.4 GB per step)"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
    return line


def run_e2e(bss, params, device, stream, steps):
    """Same metric through the public API with the inputs in pinned host memory:
    each step copies Q and the latent host->device, runs the prefill, copies O and
    LSE device->host; timed with CUDA events on the stream."""
    import torch
    q_d, lat_d, cu = make_inputs(device, seed_offset=7)
    q_h = torch.empty(q_d.shape, dtype=q_d.dtype, pin_memory=True)
    lat_h = torch.empty(lat_d.shape, dtype=lat_d.dtype, pin_memory=True)
    q_h.copy_(q_d)
    lat_h.copy_(lat_d)
    out_h = torch.empty((SEQLEN, H, DV), dtype=torch.bfloat16, pin_memory=True)
    lse_h = torch.empty((SEQLEN, H), dtype=torch.float32, pin_memory=True)
    out_d = torch.empty((SEQLEN, H, DV), dtype=torch.bfloat16, device=device)
    lse_d = torch.empty((SEQLEN, H), dtype=torch.float32, device=device)
    torch.cuda.synchronize()

    def one():
        q_d.copy_(q_h, non_blocking=True)
        lat_d.copy_(lat_h, non_blocking=True)
        bss.loza_ssa_prefill(q_d, lat_d, lat_d[:, :, :DV], cu, SEQLEN, params, out=out_d, lse=lse_d, stream=stream)
        out_h.copy_(out_d, non_blocking=True)
        lse_h.copy_(lse_d, non_blocking=True)

    one()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = q_h.numel() * 2 + lat_h.numel() * 2
    d2h = out_h.numel() * 2 + lse_h.numel() * 4
    del q_h, lat_h, out_h, lse_h, q_d, lat_d, out_d, lse_d
    return {"value": prefill_flops() / (ms / 1000.0) / 1e12, "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
