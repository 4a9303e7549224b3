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


def kernel_source_hash(files=None):
    """sha256 (first 16 hex digits) of the given csrc/ files, in sorted order,
    or of every file in csrc/ when none are given."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_streaming_b200", "csrc")
    for f in sorted(files if files else os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key, scale=1.0):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None. `scale`: this launch's units over
    those of the recorded launch, for a kernel whose traffic grows in
    proportion to them (the record says which units)."""
    p = os.path.join(ROOT, "profiles", "ncu_counters.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash(e.get("source_files")):
        return None
    return int(round(e.get("dram_bytes_per_launch") * scale))


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

_LATENT_CACHE = {}


def oracle_sample(n_rows_target_s=15.0, rank_seed=0, seq_len=SEQLEN):
    """Time the fp64 oracle on a bounded sample of the prefill workload: query rows
    spread over the sequence (all 64 heads of each). Returns (TFLOP/s, desc, cores, s)."""
    import oracle
    oracle.build()
    g = synth.rng(synth.workload_seed(2))
    L = seq_len
    # the latent KV in full (37.7 MB); Q only for the sampled rows
    if L not in _LATENT_CACHE:
        lat0 = synth.normal_bits(g, (L, 1, DQK))
        _LATENT_CACHE[L] = (lat0, np.ascontiguousarray(lat0[:, :, :DV]))
    lat, vlat = _LATENT_CACHE[L]
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
    per_step_s = max(0.5, 150.0 / (args.warmup + args.steps))   # whole run within a few minutes
    for i in range(args.warmup + args.steps):
        v, desc, cores, dt = oracle_sample(n_rows_target_s=per_step_s, rank_seed=i)
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


# --------------------------------------------------------------------------- multi-rank helpers

def max_over_ranks(x: float, device) -> float:
    """Maximum of a per-rank number over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, steps: int, work_per_step: float, max_ms: float) -> float:
    """Whole-job throughput: the work of all ranks' replicas over the slowest rank's time."""
    return world * steps * work_per_step / (max_ms / 1000.0)


# --------------------------------------------------------------------------- GPU leg

def make_inputs(device, seq_len, seed_offset=0):
    import torch
    seed = synth.workload_seed(2) * 1000 + seed_offset
    q = synth.torch_normal_bf16((seq_len, H, DQK), seed, device)
    lat = synth.torch_normal_bf16((seq_len, 1, DQK), seed + 1, device)
    cu = torch.tensor([0, seq_len], dtype=torch.int32, device=device)
    return q, lat, cu


def time_launches(fn, stream, n, flush=None):
    """Mean device time (ms) of n calls of fn, CUDA events on `stream` around each
    call only; `flush` (if given) runs before every call, outside the events."""
    import torch
    ts = []
    for _ in range(n):
        if flush is not None:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.mean(ts), ts


def time_rotating(bss, q, cache, seqlens, cap, params, ws, copies, reps=10):
    """Mean device time (ms) of one decode call when calls run back to back
    over `copies` independent copies of q, the cache and the outputs: each
    call's data was last touched copies - 1 calls earlier, with more bytes
    than L2 holds touched in between, so no flush (and none of the write-back
    a flush write leaves in L2) is needed. One pass over the copies is
    captured in a CUDA graph, so no host time separates the calls."""
    import torch
    qs = [q] + [q.clone() for _ in range(copies - 1)]
    caches = [cache] + [cache.clone() for _ in range(copies - 1)]
    outs = [torch.empty((q.shape[0], H, DV), dtype=torch.bfloat16, device=q.device) for _ in range(copies)]
    lses = [torch.empty((q.shape[0], H), dtype=torch.float32, device=q.device) for _ in range(copies)]

    def one_pass():
        for i in range(copies):
            bss.loza_ssa_decode(qs[i], caches[i], None, seqlens, cap, params, out=outs[i], lse=lses[i],
                                workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            one_pass()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    # relaxed: the library sets kernel attributes (not stream work) on every call
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        one_pass()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    e0.record(cur)
    for _ in range(reps):
        g.replay()
    e1.record(cur)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * copies)
    del g, qs, caches, outs, lses
    torch.cuda.empty_cache()
    return ms


def decode_bytes(lens, n_local=LW):
    """Algorithmic bytes of one absorbed decode call: every selected latent row once
    (576 bf16; K and V share it), q, out and lse."""
    rows = 0
    for L in lens:
        if n_local < 0:
            rows += L
        else:
            j = (L - 1) // B
            sel = set(range(min(S, j + 1))) | set(range(max(0, j - n_local + 1), j + 1))
            rows += sum(min(B, L - kb * B) for kb in sel)
    n = len(lens)
    return rows * DQK * 2 + n * H * (DQK * 2 + DV * 2 + 4)


def run_decode(bss, device, stream, lens, cap, with_dense=True, steps=20, rotating=0):
    """SSA decode (and the dense full-context decode) on a latent cache
    [len(lens), cap, 576]; L2 flushed (256 MB write, then a 256 MB read) before
    every timed call.
    rotating > 1: also time the SSA decode over that many copies of the inputs
    and outputs, back to back in a CUDA graph (time_rotating)."""
    import torch
    Bn = len(lens)
    q = synth.torch_normal_bf16((Bn, H, DQK), synth.workload_seed(3) * 1000 + 1, device)
    cache = synth.torch_normal_bf16((Bn, cap, 1, DQK), synth.workload_seed(3) * 1000 + 2, device)
    seqlens = torch.tensor(lens, dtype=torch.int32, device=device)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=device)

    def flush():
        # evict the inputs: write 256 MB, then read 256 MB more, so that the
        # write's dirty lines are written back here and not inside the timed call;
        # then keep the GPU busy for ~0.2 ms, so that the host has enqueued the
        # timed call before its start event is reached (no host time inside)
        flush_w.zero_()
        flush_r.sum()
        torch.cuda._sleep(400000)
    out = torch.empty((Bn, H, DV), dtype=torch.bfloat16, device=device)
    lse = torch.empty((Bn, H), dtype=torch.float32, device=device)
    res = {}
    for name, nl, n in (("ssa", LW, steps), ("dense", -1, 3)):
        if name == "dense" and not with_dense:
            continue
        params = bss.Params(SCALE, B, S if nl > 0 else 0, nl)
        ws = torch.empty(max(16, bss.workspace_size(bss.LOZA_OP_DECODE, Bn, 0, cap, H, 1, DQK, DV, params)),
                         dtype=torch.uint8, device=device)

        def call():
            bss.loza_ssa_decode(q, cache, None, seqlens, cap, params, out=out, lse=lse, workspace=ws, stream=stream)

        for _ in range(3):
            call()
        torch.cuda.synchronize()
        ms, _ = time_launches(call, stream, n, flush=flush)
        nbytes = decode_bytes(lens, nl)
        res[name] = {"ms": ms, "bytes": nbytes, "GB/s": nbytes / (ms / 1000.0) / 1e9, "launches_timed": n}
        if bss.device_status() != 0:
            raise RuntimeError("device status reports a timed-out wait in decode")
        if name == "ssa" and rotating > 1:
            try:
                ms_r = time_rotating(bss, q, cache, seqlens, cap, params, ws, rotating)
                res["ssa_rotating"] = {"ms": ms_r, "bytes": nbytes, "GB/s": nbytes / (ms_r / 1000.0) / 1e9,
                                       "copies": rotating}
            except RuntimeError as e:  # a secondary timing; the flushed one above stands
                torch.cuda.synchronize()
                print(f"rotating decode timing skipped: {e}", file=sys.stderr)
    del cache
    torch.cuda.empty_cache()
    return res


# the kernel the library's decode plan picks for the 1 + 7 window at these batches
DECODE_KERNEL = "ssa_decode_mla_hb_kernel"


def decode_secondary(bss, device, stream, peaks, peak_kind, batch=None, ctx=None):
    w = synth.WORKLOADS[3]
    g = synth.rng(synth.workload_seed(3))
    lo, hi = (w["ctx_lo"], w["ctx_hi"]) if ctx is None else (ctx // 2, ctx)
    lens = synth.uniform_lengths(g, w["batch"], lo, hi).tolist()
    if batch is not None:
        lens = lens[:batch]
    r = run_decode(bss, device, stream, lens, hi, rotating=4)
    hbm = float(peaks["hbm_gbs"])
    ssa = r["ssa"]
    name = w["name"] if len(lens) == w["batch"] else f"{w['name']} (first {len(lens)} sequences)"
    if ctx is not None:
        name += f" (contexts in [{lo}, {hi}])"
    out = {"workload": name,
           "metric": "SSA decode GB/s (bytes touched)", "value": ssa["GB/s"], "unit": "GB/s",
           "ms_per_call": ssa["ms"], "bytes_per_call": ssa["bytes"],
           "roofline": {"bound": "hbm", "achieved": ssa["GB/s"], "peak": hbm, "unit": "GB/s",
                        "frac": ssa["GB/s"] / hbm,
                        "traffic": profiled_traffic(DECODE_KERNEL, len(lens) / w["batch"]),
                        "peak_kind": f"{peak_kind} HBM copy (MEASURED_PEAKS.json hbm_gbs)",
                        "kernel": DECODE_KERNEL},
           "timing": "mean of per-call CUDA events; before each call (outside the events) the L2 is flushed "
                     "by a 256 MB write and then a 256 MB read, so the call starts with no dirty lines to write "
                     "back, and a ~0.2 ms device sleep keeps the start event from waiting on the host"}
    if "ssa_rotating" in r:
        rr = r["ssa_rotating"]
        out["rotating"] = {"ms_per_call": rr["ms"], "GB/s": rr["GB/s"], "frac_of_hbm": rr["GB/s"] / hbm,
                           "timing": f"calls back to back over {rr['copies']} copies of q, cache and outputs "
                                     "(more than L2 touched between two uses of a copy; no flush), one pass "
                                     "over the copies captured in a CUDA graph, mean over 10 replays"}
    if "dense" in r:
        d = r["dense"]
        out["dense"] = {"ms_per_call": d["ms"], "bytes_per_call": d["bytes"], "GB/s": d["GB/s"],
                        "frac_of_hbm": d["GB/s"] / hbm, "ssa_speedup": d["ms"] / ssa["ms"]}
    return out


def prefill_workspace(bss, device, batch, T, L, params, H_=None, Hkv=1, dqk=None, dv=None):
    """Device workspace for loza_ssa_prefill, allocated once outside the timed
    region (None when the shape needs none)."""
    import torch
    n = bss.workspace_size(bss.LOZA_OP_PREFILL, batch, T, L, H_ or H, Hkv, dqk or DQK, dv or DV, params)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def merge_secondary(bss, device, stream, peaks, peak_kind, steps=20):
    """LSE merge of two attention branches (O, LSE) at the prefill's output
    shape: 32,768 tokens x 64 heads x 512 values. Inputs are 4.3 GB (> L2)."""
    import torch
    rows, d_v = SEQLEN * H, DV
    o_a = synth.torch_normal_bf16((rows, d_v), 9001, device)
    o_b = synth.torch_normal_bf16((rows, d_v), 9002, device)
    g = torch.Generator(device=device).manual_seed(9003)
    l_a = torch.rand(rows, device=device, generator=g) * 25 - 5
    l_b = torch.rand(rows, device=device, generator=g) * 25 - 5
    out = torch.empty_like(o_a)
    lse = torch.empty_like(l_a)

    def call():
        bss.loza_ssa_merge(o_a, l_a, o_b, l_b, out=out, lse_out=lse, stream=stream)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms, _ = time_launches(call, stream, steps)
    nbytes = rows * (3 * d_v * 2 + 3 * 4)
    hbm = float(peaks["hbm_gbs"])
    gbs = nbytes / (ms / 1000.0) / 1e9
    del o_a, o_b, out
    torch.cuda.empty_cache()
    return {"workload": f"merge of two attention branches, {SEQLEN} tokens x {H} heads x {DV}",
            "metric": "branch merge GB/s", "value": gbs, "unit": "GB/s", "ms_per_call": ms,
            "bytes_per_call": nbytes,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "traffic": profiled_traffic("ssa_merge_kernel"),
                         "peak_kind": f"{peak_kind} HBM copy (MEASURED_PEAKS.json hbm_gbs)",
                         "kernel": "ssa_merge_kernel"},
            "timing": "mean of per-call CUDA events; inputs larger than L2"}


def tensor_roofline(flop, ms, peaks, peak_kind, kernel, traffic_scale=1.0, sustained=False):
    """sustained: the kernel runs for tens of milliseconds per launch, back to
    back, so it is held to the sustained (power-capped) GEMM figure; the
    fraction of the burst figure is reported beside it."""
    burst = float(peaks["bf16_tflops"])
    pk = float(peaks["bf16_tflops_sustained"]) if sustained else burst
    a = flop / (ms / 1000.0) / 1e12
    kind = ("bf16 dense sustained (MEASURED_PEAKS.json bf16_tflops_sustained; launches of tens of ms back to "
            "back run under the power cap)" if sustained else "bf16 dense burst (MEASURED_PEAKS.json bf16_tflops)")
    r = {"bound": "tensor", "achieved": a, "peak": pk, "unit": "TFLOP/s", "frac": a / pk,
         "traffic": profiled_traffic(kernel, traffic_scale), "peak_kind": f"{peak_kind} {kind}", "kernel": kernel}
    if sustained:
        r["frac_of_burst"] = a / burst
    return r


def hbm_roofline(nbytes, ms, peaks, peak_kind, kernel, traffic_scale=1.0):
    hbm = float(peaks["hbm_gbs"])
    a = nbytes / (ms / 1000.0) / 1e9
    return {"bound": "hbm", "achieved": a, "peak": hbm, "unit": "GB/s", "frac": a / hbm,
            "traffic": profiled_traffic(kernel, traffic_scale),
            "peak_kind": f"{peak_kind} HBM copy (MEASURED_PEAKS.json hbm_gbs)", "kernel": kernel}


def long_secondary(bss, device, stream, peaks, peak_kind):
    """Workload 4: L = 262144 absorbed prefill, SSA next to full causal attention
    (the same library, unbounded window); then SSA and dense decode of 32
    sequences of 1,048,576 tokens."""
    import torch
    w = synth.WORKLOADS[4]
    L = w["seqlen"]
    q, lat, cu = make_inputs(device, L, seed_offset=40)
    out = torch.empty((L, H, DV), dtype=torch.bfloat16, device=device)
    lse = torch.empty((L, H), dtype=torch.float32, device=device)
    lines = {}
    for name, nl, warm, n in (("ssa", LW, 2, 5), ("dense", -1, 0, 1)):
        params = bss.Params(SCALE, B, S if nl > 0 else 0, nl)
        ws = prefill_workspace(bss, device, 1, L, L, params)

        def call():
            bss.loza_ssa_prefill(q, lat, lat[:, :, :DV], cu, L, params, out=out, lse=lse, workspace=ws, stream=stream)

        for _ in range(warm):
            call()
        torch.cuda.synchronize()
        ms, _ = time_launches(call, stream, n)
        if bss.device_status() != 0:
            raise RuntimeError("device status reports a timed-out wait in the long prefill")
        fl = prefill_flops(L) if nl > 0 else 2.0 * (DQK + DV) * H * L * (L + 1) / 2
        # the library's choice for these shapes: the two-pass kernel needs a
        # workspace and a bounded window, the unbounded window runs on the pair kernel
        kern = "ssa_prefill_mla_kernel" if (nl > 0 and ws is not None) else "ssa_prefill_pair_kernel"
        lines[name] = {"ms_per_call": ms, "launches_timed": n, "algorithmic_tflop": fl / 1e12,
                       "TFLOP/s": fl / (ms / 1000) / 1e12,
                       "roofline": tensor_roofline(fl, ms, peaks, peak_kind, kern, traffic_scale=L / SEQLEN,
                                                   sustained=True)}
        del ws
    del q, lat, out, lse
    torch.cuda.empty_cache()
    res = {"workload": "MLA-absorbed SSA prefill L=262144 (64 heads, latent 576, V = first 512)",
           "metric": "SSA prefill TFLOP/s", "value": lines["ssa"]["TFLOP/s"], "unit": "TFLOP/s",
           "ms_per_call": lines["ssa"]["ms_per_call"], "roofline": lines["ssa"]["roofline"],
           "dense": dict(lines["dense"], dense_over_ssa_time=lines["dense"]["ms_per_call"] / lines["ssa"]["ms_per_call"],
                         algorithmic_ratio=lines["dense"]["algorithmic_tflop"] / lines["ssa"]["algorithmic_tflop"]),
           "timing": "mean of per-call CUDA events (SSA: 2 warm-up, 5 timed; dense: 1 timed launch of ~5 s); "
                     "inputs larger than L2"}
    r = run_decode(bss, device, stream, [w["decode_ctx"]] * w["decode_batch"], w["decode_ctx"])
    ssa, dense = r["ssa"], r["dense"]
    dec = {"workload": f"MLA-absorbed SSA decode, {w['decode_batch']} seqs x {w['decode_ctx']} tokens",
           "metric": "SSA decode GB/s (bytes touched)", "value": ssa["GB/s"], "unit": "GB/s",
           "ms_per_call": ssa["ms"], "bytes_per_call": ssa["bytes"],
           "roofline": hbm_roofline(ssa["bytes"], ssa["ms"], peaks, peak_kind, DECODE_KERNEL,
                                    traffic_scale=w["decode_batch"] / synth.WORKLOADS[3]["batch"]),
           "dense": {"ms_per_call": dense["ms"], "bytes_per_call": dense["bytes"], "GB/s": dense["GB/s"],
                     "frac_of_hbm": dense["GB/s"] / float(peaks["hbm_gbs"]),
                     "dense_over_ssa_time": dense["ms"] / ssa["ms"]},
           "timing": "mean of per-call CUDA events; L2 flushed (256 MB write, then 256 MB read) before each call"}
    return res, dec


HI_WINDOW = (1, 16, 1024)   # page 4: 16 sink tokens and a 1,024-token window (b = 1)
HI_TOP_PAGES, HI_TOP_K, HI_DIM = 1024, 1024, 128


def token_window_rows(L, win=HI_WINDOW):
    b, s, l = win
    i = L - 1
    lo = max(0, (i // b - l + 1) * b)
    return min(s * b, L) + (L - max(lo, min(s * b, L)))


def hi_secondary(bss, device, stream, peaks, peak_kind, batch=32, ctx=1 << 20, steps=10):
    """Hierarchical index decode (page 4): 32 sequences of 1,048,576 tokens,
    16 sink tokens + a 1,024-token window + 1,024 tokens selected from the top
    1,024 pages of 128, index keys of 128 bf16. Times the whole call and, apart,
    its two parts (the selection; the attention over the window and the
    selection), and the window alone for comparison; the page keys are
    maintained as the cache fills and are computed once, outside the step."""
    import torch
    seed = synth.workload_seed(4) * 1000 + 70
    q = synth.torch_normal_bf16((batch, H, DQK), seed, device)
    cache = synth.torch_normal_bf16((batch, ctx, 1, DQK), seed + 1, device)
    k_idx = synth.torch_normal_bf16((batch, ctx, HI_DIM), seed + 2, device)
    q_idx = synth.torch_normal_bf16((batch, HI_DIM), seed + 3, device)
    lens = [ctx] * batch
    seqlens = torch.tensor(lens, dtype=torch.int32, device=device)
    params = bss.Params(SCALE, *HI_WINDOW)
    pk = bss.loza_hi_page_keys(k_idx, seqlens, ctx, stream=stream)
    out = torch.empty((batch, H, DV), dtype=torch.bfloat16, device=device)
    lse = torch.empty((batch, H), dtype=torch.float32, device=device)
    o_w = torch.empty_like(out)
    l_w = torch.empty_like(lse)
    ws = torch.empty(max(16, bss.hi_workspace_size(batch, ctx, HI_TOP_PAGES, HI_TOP_K, params)), dtype=torch.uint8,
                     device=device)
    ws_sel = torch.empty(max(16, bss.hi_workspace_size(batch, ctx, 1, HI_TOP_K, params)), dtype=torch.uint8,
                         device=device)
    ws_dec = torch.empty(max(16, bss.workspace_size(bss.LOZA_OP_DECODE, batch, 0, ctx, H, 1, DQK, DV, params)),
                         dtype=torch.uint8, device=device)
    sel = torch.empty((batch, HI_TOP_K), dtype=torch.int32, device=device)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=device)

    def flush():
        flush_w.zero_()
        flush_r.sum()
        torch.cuda._sleep(400000)

    calls = {
        "hi_decode": lambda: bss.loza_hi_decode(q, cache, q_idx, k_idx, pk, seqlens, ctx, params, HI_TOP_PAGES,
                                                HI_TOP_K, out=out, lse=lse, workspace=ws, stream=stream),
        "select": lambda: bss.loza_hi_select(q_idx, k_idx, pk, seqlens, ctx, params, HI_TOP_PAGES, HI_TOP_K,
                                             selected=sel, workspace=ws, stream=stream),
        "decode_selected": lambda: bss.loza_ssa_decode_selected(q, cache, seqlens, ctx, params, sel, out=o_w,
                                                                lse=l_w, workspace=ws_sel, stream=stream),
        "window_only_decode": lambda: bss.loza_ssa_decode(q, cache, None, seqlens, ctx, params, out=o_w, lse=l_w,
                                                          workspace=ws_dec, stream=stream),
        "page_keys": lambda: bss.loza_hi_page_keys(k_idx, seqlens, ctx, page_keys=pk, stream=stream),
    }
    ms = {}
    launches = {}
    for name, fn in calls.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        c0 = bss.launch_count()
        ms[name], _ = time_launches(fn, stream, steps if name != "page_keys" else 3, flush=flush)
        launches[name] = (bss.launch_count() - c0) // (steps if name != "page_keys" else 3)
    if bss.device_status() != 0:
        raise RuntimeError("device status reports a timed-out wait in the HI decode")
    # algorithmic bytes of one step
    n_pages = ctx // 128
    b_select = batch * (n_pages * HI_DIM * 4 + HI_TOP_PAGES * 128 * HI_DIM * 2 + HI_DIM * 2)
    b_attend = batch * ((token_window_rows(ctx) + HI_TOP_K) * DQK * 2 + H * (DQK * 2 + DV * 2 + 4))
    total = b_select + b_attend
    dense_bytes = batch * (ctx * DQK * 2 + H * (DQK * 2 + DV * 2 + 4))
    parts = {"select": b_select, "decode_selected": b_attend,
             "window_only_decode": batch * (token_window_rows(ctx) * DQK * 2 + H * (DQK * 2 + DV * 2 + 4))}
    del q, cache, k_idx, q_idx, pk, ws, ws_sel, ws_dec
    torch.cuda.empty_cache()
    hbm = float(peaks["hbm_gbs"])
    gbs = total / (ms["hi_decode"] / 1000.0) / 1e9
    return {"workload": f"hierarchical index decode (MLA-absorbed), {batch} seqs x {ctx} tokens, "
                        f"window 16 sink + 1,024 tokens, top {HI_TOP_PAGES} pages of 128, top {HI_TOP_K} tokens, "
                        f"index keys {HI_DIM} bf16",
            "metric": "HI decode GB/s (bytes touched)", "value": gbs, "unit": "GB/s",
            "ms_per_call": ms["hi_decode"], "bytes_per_call": total, "launches_per_call": launches["hi_decode"],
            "roofline": hbm_roofline(total, ms["hi_decode"], peaks, peak_kind, "hi_decode (all its kernels)"),
            "parts": {k: {"ms_per_call": ms[k], "bytes_per_call": parts[k],
                          "GB/s": parts[k] / (ms[k] / 1000.0) / 1e9,
                          "frac_of_hbm": parts[k] / (ms[k] / 1000.0) / 1e9 / hbm, "launches": launches[k]}
                      for k in parts},
            "page_keys_once": {"ms": ms["page_keys"], "bytes": batch * (ctx * HI_DIM * 2 + n_pages * HI_DIM * 4)},
            "dense_decode_bytes_per_call": dense_bytes,
            "timing": "mean of per-call CUDA events; L2 flushed (256 MB write, then 256 MB read) and a ~0.2 ms "
                      "device sleep before each call"}


def train_secondary(bss, device, stream, peaks, peak_kind, train_len=None):
    """Workload 5: varlen forward + backward, per-head 192/128 dims, 64 heads
    (train_len: one sequence of that many tokens instead, for profiling)."""
    import torch
    w = synth.WORKLOADS[5]
    g = synth.rng(synth.workload_seed(5))
    lens = synth.loguniform_lengths(g, w["batch"], w["len_lo"], w["len_hi"], w["total_cap"])
    if train_len:
        lens = np.array([train_len], dtype=np.int64)
    T = int(lens.sum())
    Hh, dqk, dv = w["n_heads"], w["d_qk"], w["d_v"]
    base = synth.workload_seed(5) * 1000
    q = synth.torch_normal_bf16((T, Hh, dqk), base + 1, device)
    k = synth.torch_normal_bf16((T, Hh, dqk), base + 2, device)
    v = synth.torch_normal_bf16((T, Hh, dv), base + 3, device)
    do = synth.torch_normal_bf16((T, Hh, dv), base + 4, device)
    cu = torch.from_numpy(synth.cu_seqlens(lens)).to(device)
    params = bss.Params(w["scale"], B, S, LW)
    out = torch.empty((T, Hh, dv), dtype=torch.bfloat16, device=device)
    lse = torch.empty((T, Hh), dtype=torch.float32, device=device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dvv = torch.empty_like(v)
    ws = torch.empty(bss.workspace_size(bss.LOZA_OP_BACKWARD, len(lens), T, int(lens.max()), Hh, Hh, dqk, dv, params),
                     dtype=torch.uint8, device=device)
    pairs = sum(visible_pairs(int(L)) for L in lens)
    f_fwd = 2.0 * (dqk + dv) * Hh * pairs
    f_bwd = 2.0 * (3 * dqk + 2 * dv) * Hh * pairs

    def fwd():
        bss.loza_ssa_prefill(q, k, v, cu, int(lens.max()), params, out=out, lse=lse, stream=stream)

    def bwd():
        bss.loza_ssa_backward(q, k, v, out, do, lse, cu, int(lens.max()), params, dq=dq, dk=dk, dv=dvv,
                              workspace=ws, stream=stream)

    for _ in range(3):
        fwd()
        bwd()
    torch.cuda.synchronize()
    mf, _ = time_launches(fwd, stream, 5)
    mb, _ = time_launches(bwd, stream, 5)
    if bss.device_status() != 0:
        raise RuntimeError("device status reports a timed-out wait in training")
    name = w["name"] if not train_len else f"training fwd+bwd, one sequence of {train_len} tokens"
    res = {"workload": f"{name}, {Hh} heads, q/k {dqk}, v {dv}", "lengths": lens.tolist(), "total_tokens": T,
           "metric": "SSA training TFLOP/s (forward, backward)", "unit": "TFLOP/s",
           "value": (f_fwd + f_bwd) / ((mf + mb) / 1000) / 1e12,
           "forward": {"ms_per_call": mf, "TFLOP/s": f_fwd / (mf / 1000) / 1e12, "algorithmic_tflop": f_fwd / 1e12,
                       "roofline": tensor_roofline(f_fwd, mf, peaks, peak_kind, "ssa_prefill_mha2_kernel",
                                                   sustained=True)},
           "backward": {"ms_per_call": mb, "TFLOP/s": f_bwd / (mb / 1000) / 1e12, "algorithmic_tflop": f_bwd / 1e12,
                        "roofline": tensor_roofline(f_bwd, mb, peaks, peak_kind, "ssa_bwd", sustained=True),
                        "flop_per_pair_head": 2 * (3 * dqk + 2 * dv)},
           "timing": "mean of per-call CUDA events, 3 warm-up and 5 timed calls each; inputs larger than L2"}
    del q, k, v, do, out, lse, dq, dk, dvv, ws
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import block_sparse_streaming_b200 as bss

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    bss.lib()
    stream = torch.cuda.current_stream()
    peaks, peak_kind = measured_peaks()
    L = args.seq_len
    params = bss.Params(SCALE, B, S, LW)
    q, lat, cu = make_inputs(device, L, seed_offset=rank)
    v = lat[:, :, :DV]
    out = torch.empty((L, H, DV), dtype=torch.bfloat16, device=device)
    lse = torch.empty((L, H), dtype=torch.float32, device=device)
    ws = prefill_workspace(bss, device, 1, L, L, params)

    def step():
        bss.loza_ssa_prefill(q, lat, v, cu, L, params, out=out, lse=lse, workspace=ws, stream=stream)

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
    if bss.device_status() != 0:
        raise RuntimeError("device status reports a timed-out wait after the timed region")
    del q, lat, out, lse
    torch.cuda.empty_cache()

    total_ms = max_over_ranks(total_ms, device)
    flops = prefill_flops(L)
    value = job_value(world, args.steps, flops, total_ms) / 1e12

    e2e = None if args.no_e2e else run_e2e(bss, params, device, stream, L, steps=max(1, min(args.steps, 3)))
    if e2e is not None and world > 1:
        # whole job, as `value`: every rank's replica over the slowest rank's time
        ms = max_over_ranks(e2e["ms_per_step"], device)
        e2e.update(ms_per_step=ms, value=job_value(world, 1, prefill_flops(L), ms) / 1e12,
                   h2d_bytes_per_step=world * e2e["h2d_bytes_per_step"],
                   d2h_bytes_per_step=world * e2e["d2h_bytes_per_step"])

    avg_launch_ms = statistics.mean(per_launch_ms)
    achieved = flops / (avg_launch_ms / 1000.0) / 1e12
    peak = float(peaks["bf16_tflops"])
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": profiled_traffic("ssa_prefill_mla_kernel"),
                "peak_kind": f"{peak_kind} bf16 dense burst (MEASURED_PEAKS.json bf16_tflops)",
                "kernel": "ssa_prefill_mla_kernel",
                "algorithmic_flop_per_launch": flops,
                "avg_launch_ms": avg_launch_ms}

    secondary = {}
    if args.workload in ("default", "decode"):
        secondary["decode"] = decode_secondary(bss, device, stream, peaks, peak_kind, args.decode_batch,
                                               args.decode_ctx)
    if args.workload in ("default", "merge"):
        secondary["merge"] = merge_secondary(bss, device, stream, peaks, peak_kind)
    if args.workload in ("default", "long"):
        secondary["long"], secondary["decode_1m"] = long_secondary(bss, device, stream, peaks, peak_kind)
    if args.workload in ("default", "hi"):
        secondary["hi_decode"] = hi_secondary(bss, device, stream, peaks, peak_kind, args.hi_batch, args.hi_ctx)
    if args.workload in ("default", "train"):
        secondary["train"] = train_secondary(bss, device, stream, peaks, peak_kind, args.train_len)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v_cpu, desc, cores, _ = oracle_sample(seq_len=L)
            cpu = {"value": v_cpu, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD["name"] if L == SEQLEN else f"MLA-absorbed SSA prefill L={L}",
                       "batch": 1, "seq_len": L, "n_heads": H,
                       "kv": "shared latent 576 (V = first 512)", "d_qk": DQK, "d_v": DV,
                       "block": [B, S, LW], "parallelism": f"replica x{world}",
                       "l2": f"inputs larger than L2 (Q is {L * H * DQK * 2 / 1e9:.2f} GB per step)"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "secondary": secondary,
        }
    return line


def run_e2e(bss, params, device, stream, L, steps):
    """Same metric through the public C-ABI call with HOST buffers
    (loza_ssa_prefill_host): every step copies Q and the latent from pinned host
    memory to the device and O and LSE back, inside the call, pipelined over
    chunks of query blocks; timed with CUDA events on the stream the call
    completes on."""
    import torch
    q_d, lat_d, cu = make_inputs(device, L, seed_offset=7)
    q_h = torch.empty(q_d.shape, dtype=q_d.dtype, pin_memory=True)
    lat_h = torch.empty(lat_d.shape, dtype=lat_d.dtype, pin_memory=True)
    q_h.copy_(q_d)
    lat_h.copy_(lat_d)
    del q_d, lat_d
    torch.cuda.empty_cache()
    out_h = torch.empty((L, H, DV), dtype=torch.bfloat16, pin_memory=True)
    lse_h = torch.empty((L, H), dtype=torch.float32, pin_memory=True)
    ws = torch.empty(bss.workspace_size(bss.LOZA_OP_PREFILL_HOST, 1, L, L, H, 1, DQK, DV, params), dtype=torch.uint8,
                     device=device)
    torch.cuda.synchronize()

    def one():
        bss.loza_ssa_prefill_host(q_h, lat_h, lat_h[:, :, :DV], params, out=out_h, lse=lse_h, workspace=ws,
                                  stream=stream)

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
    del ws
    torch.cuda.empty_cache()
    floor = copy_floor_ms(stream, [q_h, lat_h], [out_h, lse_h], steps)
    del q_h, lat_h, out_h, lse_h
    torch.cuda.empty_cache()
    return {"value": prefill_flops(L) / (ms / 1000.0) / 1e12, "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "api": "loza_ssa_prefill_host",
            "copy_floor_ms": floor, "frac_of_copy_floor": floor / ms,
            "copy_floor": "the same host<->device bytes alone, both directions at once on two streams, no kernels"}


def copy_floor_ms(stream, host_in, host_out, steps):
    """Time of the step's PCIe traffic alone: the pinned inputs copied to the
    device while same-sized device buffers are copied to the pinned outputs,
    on two streams; the e2e step cannot be faster than this."""
    import torch
    dev_in = [torch.empty_like(t, device="cuda") for t in host_in]
    dev_out = [torch.empty_like(t, device="cuda") for t in host_out]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def one():
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        with torch.cuda.stream(s_in):
            for d, h in zip(dev_in, host_in):
                d.copy_(h, non_blocking=True)
        with torch.cuda.stream(s_out):
            for h, d in zip(host_out, dev_out):
                h.copy_(d, non_blocking=True)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

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
    del dev_in, dev_out
    return ms


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--seq-len", type=int, default=SEQLEN,
                    help="prefill length (default: the 32,768-token workload; smaller values serve profiling)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="use only the first N sequences of the decode workload (profiling)")
    ap.add_argument("--decode-ctx", type=int, default=None,
                    help="decode contexts in [N/2, N] instead of the workload's (profiling: same bytes per "
                         "sequence, a smaller cache)")
    ap.add_argument("--train-len", type=int, default=None,
                    help="training workload as one sequence of this length (profiling)")
    ap.add_argument("--hi-batch", type=int, default=32, help="sequences of the hierarchical index decode line")
    ap.add_argument("--hi-ctx", type=int, default=1 << 20, help="tokens per sequence of that line (a multiple of 128)")
    ap.add_argument("--workload", choices=["default", "prefill", "decode", "merge", "long", "hi", "train"], default="default",
                    help="default: the prefill line with every other workload as secondary lines (the "
                         "64-sequence decode, the branch merge, workload 4's long prefill and 1M decode, "
                         "the hierarchical index decode at 1M, workload 5's training); the others: the prefill line plus only that one")
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
