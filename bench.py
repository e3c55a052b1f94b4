#!/usr/bin/env python
"""Benchmark of the sparse MoE expert layer on B200.

Default workload (the headline): one Flash-Next-shaped MoE layer in decode,
d=2048, f=768, E=512, top-10 renormalised softmax + 1 shared expert,
4-bit symmetric group-32 experts, bf16 hidden N(0,1), verify window T=4,
uniform routing.  A step = one moe_forward call (router, top-k, residency
lookup, bucketing, dequant-SwiGLU experts, combine + residual) on a new
4-token window.  Steps rotate over --rot-layers independent copies of the
layer's weights (16 x 1.36 GB by default), so the weights a step reads were
evicted from the 126 MB L2 long before (no flush needed).

Other workloads: --workload q2 (2-bit asymmetric g64, Zipf(1.1) routing,
64 sequences x T tokens per call), --workload prefill (8192-token chunk).

Contract: python bench.py --gpus N --steps K --warmup W [--impl reference];
rank 0 prints one JSON line.  N > 1 runs N independent replicas (the layer
does not shard; no collective on the data path), value = all ranks' tokens /
max-over-ranks time.
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

D, F, E, K_TOP = 2048, 768, 512, 10


def parse():
    ap = argparse.ArgumentParser()
    # (defaults that depend on the workload are filled in below)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 200 decode windows, 20 prefill chunks)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "q2", "prefill", "stack"])
    ap.add_argument("--T", type=int, default=4, help="window (decode) / per-sequence window (q2)")
    ap.add_argument("--rot-layers", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args()
    if a.steps is None:
        a.steps = {"prefill": 20, "stack": 10}.get(a.workload, 200)
    return a


# ----------------------------------------------------------------- helpers
def kernel_traffic(kernel_bytes_per_launch):
    """Per-launch DRAM traffic of decode_kernel from the committed ncu record,
    scaled to this run's algorithmic bytes per launch (the record's launch
    routed a different window).  None when the kernel sources changed since
    the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        rec = json.load(fh)
    h = hashlib.sha256()
    for s in rec["sources"]:
        with open(os.path.join(ROOT, s), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != rec["sources_sha256"]:
        return None
    return rec["traffic_over_algorithmic"] * kernel_bytes_per_launch


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    """One process per GPU (torchrun env).  NCCL on GPUs; gloo where there is
    no GPU (the host-side logic's CPU tests)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=300)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, units_per_rank, ms_max):
    """Units all ranks processed (replicas: the same per rank) over the
    slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


# ------------------------------------------------------------ the workload
def workload_spec(args):
    from sparse_moe_expert_gemv_b200 import inputs as I
    if args.workload == "decode":
        return dict(name=f"one MoE layer decode, d=2048 f=768 E=512 top-10 + shared, Q4 g32, "
                         f"T={args.T}, uniform routing", fmt=I.Q4, zipf=False, T=args.T, seqs=1)
    if args.workload == "q2":
        return dict(name=f"one MoE layer decode, Q2 g64 asym, Zipf(1.1) routing, 64 sequences x "
                         f"T={args.T}", fmt=I.Q2, zipf=True, T=args.T * 64, seqs=64)
    if args.workload == "stack":
        return dict(name="48-layer MoE stack (RMSNorm -> router -> experts -> combine + residual), "
                         "d=2048 f=768 E=512 top-10 + shared, Q4 g32, 4096-slot residency table by "
                         "Zipf rank, Zipf(1.1) routing, T=4 x batch 8 = 32 tokens",
                    fmt=I.Q4, zipf=True, T=32, seqs=8)
    return dict(name="prefill chunk, 8192 tokens, one MoE layer, Q4 g32, Zipf(1.1) routing",
                fmt=I.Q4, zipf=True, T=8192, seqs=1)


def build_native(args, spec, n_rot):
    import torch
    from sparse_moe_expert_gemv_b200 import binding as B
    from sparse_moe_expert_gemv_b200 import inputs as I
    ctx = B.moe_create(D, F, E, K_TOP, spec["fmt"])
    B.moe_configure(ctx, n_rot, 1, 0, spec["T"])
    for l in range(n_rot):
        W = I.router_np(args.seed, E, D, l)
        bias = I.zipf_bias_np(args.seed, E, l)[0] if spec["zipf"] else None
        B.moe_set_router(ctx, l, W, bias)
        for first in range(0, E, 64):
            c, s, m = I.experts_torch(args.seed, spec["fmt"], D, F, l, first, 64, "cuda")
            B.moe_load_experts(ctx, l, first, 64, c, s, m)
            del c, s, m
        c, s, m = I.shared_np(args.seed, spec["fmt"], D, F, l)
        B.moe_load_shared(ctx, l, c, s, m)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return ctx


def run_native(args, world, rank, local):
    import torch
    from sparse_moe_expert_gemv_b200 import binding as B
    from sparse_moe_expert_gemv_b200 import inputs as I

    spec = workload_spec(args)
    T = spec["T"]
    n_rot = args.rot_layers
    K, W = args.steps, args.warmup
    ctx = build_native(args, spec, n_rot)
    Be = B.moe_expert_bytes(D, F, spec["fmt"])

    # one fresh window per step (timed and warm-up), pristine copies kept
    n_win = K + W
    xs = np.stack([I.hidden_np(args.seed, T, D, window=i) for i in range(n_win)])
    x_host = torch.from_numpy(xs.view(np.int16)).pin_memory()
    x_dev0 = x_host.cuda()
    x_work = x_dev0.clone()
    layer_of = [i % n_rot for i in range(n_win)]

    # routing pre-pass (untimed): distinct experts each timed step touches
    idx = torch.empty((T, K_TOP), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, K_TOP), dtype=torch.float32, device="cuda")
    distinct = []
    for i in range(W, n_win):
        B.moe_route(ctx, layer_of[i], x_dev0[i], T, idx, wts)
        distinct.append(len(np.unique(idx.cpu().numpy())))
    distinct = np.array(distinct)
    expert_bytes = float((distinct + 1).sum() * Be)          # routed + shared
    router_bytes = float(K * E * D * 4)
    act_bytes = float(K * (T * D * 2 * 2))                      # x read + x written
    total_bytes = expert_bytes + router_bytes + act_bytes

    stream = torch.cuda.current_stream()
    prefill = args.workload == "prefill"
    call = B.moe_prefill if prefill else B.moe_forward  # the public call a step makes
    # warm-up (eager), then capture the K timed steps as one CUDA graph
    for i in range(W):
        call(ctx, layer_of[i], x_work[i], T)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(W, n_win):
            call(ctx, layer_of[i], x_work[i], T)
    torch.cuda.synchronize()
    x_work.copy_(x_dev0)
    torch.cuda.synchronize()
    g.replay()  # one untimed replay (graph upload, clocks)
    x_work.copy_(x_dev0)
    torch.cuda.synchronize()

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(world, ms)
    clocks = clk.summary()

    # profiled pass (same steps, CUDA events around each segment)
    B.moe_set_profiling(ctx, 1)
    gp = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gp):
        for i in range(W, n_win):
            call(ctx, layer_of[i], x_work[i], T)
    x_work.copy_(x_dev0)
    torch.cuda.synchronize()
    gp.replay()
    route_ms, exp_ms, comb_ms, ncalls = B.moe_read_profile(ctx)
    B.moe_set_profiling(ctx, 0)

    # end to end through the public call with host buffers: every step copies
    # its window in from pinned host memory and its result back out.  The
    # copies run on a second stream with two device buffers, so step i's
    # read-back and step i+1's input overlap step i's kernel; every copy is
    # inside the timed region.
    out_host = torch.empty_like(x_host).pin_memory()
    cs = torch.cuda.Stream()
    bufs = [torch.empty((T, D), dtype=torch.int16, device="cuda") for _ in range(2)]
    h2d = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]

    def put(i):
        with torch.cuda.stream(cs):
            bufs[i % 2].copy_(x_host[i], non_blocking=True)
            h2d[i % 2].record(cs)

    def run_steps(first, last):
        put(first)
        for i in range(first, last):
            if i + 1 < last:
                put(i + 1)  # its buffer's previous read-back is earlier on cs
            stream.wait_event(h2d[i % 2])
            call(ctx, layer_of[i], bufs[i % 2], T)
            done[i % 2].record(stream)
            with torch.cuda.stream(cs):
                cs.wait_event(done[i % 2])
                out_host[i].copy_(bufs[i % 2], non_blocking=True)

    run_steps(0, min(W, 3))
    torch.cuda.synchronize()
    barrier(world)
    e0.record(cs)
    run_steps(W, n_win)
    e1.record(cs)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, e0.elapsed_time(e1))
    B.moe_sync(ctx, 60000)

    hbm, tflops, peak_kind = peaks()
    tok = T * K
    # windows of <= 32 tokens run as one decode_kernel launch per step (the
    # profile's three segments are then one kernel); larger ones as five
    # launches, of which the two expert GEMV launches dominate
    single = T <= 32
    flops = 6.0 * D * F * (T * K_TOP + T)  # per call: gate, up, down GEMMs, routed + shared rows
    if prefill:
        gemm_ms = exp_ms / max(ncalls, 1)  # the two grouped GEMM launches of one call
        gemm_tf = flops / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
    if single:
        # the timed graph holds exactly one decode_kernel launch per step and
        # nothing else, so its device time over K launches is the kernel's;
        # the event-bracketed profile pass (events between launches break the
        # programmatic overlap of consecutive launches) is reported beside it
        kern_ms = ms_max
        bracketed_us = (route_ms + exp_ms + comb_ms) / max(ncalls, 1) * 1e3
        kern_bytes = expert_bytes + router_bytes
        kern_name = "decode_kernel (the whole layer: router, routing, gate/up, down, combine)"
        per_unit = (f"{Be} B per touched expert (codes+scales, shared expert included) "
                    f"+ {E * D * 4} B router W per launch")
    else:
        kern_ms = exp_ms
        kern_bytes = expert_bytes
        kern_name = "expert_gemv_kernel (gate/up + down launches of one call)"
        per_unit = f"{Be} B per touched expert (codes+scales), shared expert included"
    kern_gbs = kern_bytes / (kern_ms * 1e-3) / 1e9 if kern_ms > 0 else None
    res = {
        "metric": "decode MoE tokens/s" if args.workload != "prefill" else "prefill MoE tokens/s",
        "value": whole_job_rate(world, tok, ms_max),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_max / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("q4-g32 weights dequantised to fp16 per tile, fp16 activations, fp32 accumulate"
                  if prefill else
                  "q4-g32 weights, bf16 activations, fp32 accumulate" if spec["fmt"] == I.Q4
                  else "q2-g64 weights, bf16 activations, fp32 accumulate"),
        "data": "synthetic (seeded generator; random-init weights of the layer's shape)",
        "config": {"workload": spec["name"], "tokens_per_step": T, "layers_rotated": n_rot,
                   "l2": f"no flush: each step reads a different layer copy "
                         f"({n_rot} x {E * Be / 1e9:.2f} GB >> 126 MB L2)",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "timing": "one CUDA-graph replay of the K steps, CUDA events"},
        "expert_weight_gbs": expert_bytes / (ms_max * 1e-3) / 1e9,
        "step_gbs": total_bytes / (ms_max * 1e-3) / 1e9,
        "distinct_experts_per_step": float(distinct.mean()),
        "segments_ms_per_step": {"route": route_ms / max(ncalls, 1),
                                 "experts": exp_ms / max(ncalls, 1),
                                 "combine": comb_ms / max(ncalls, 1)},
        "roofline": {
            "bound": "tensor",
            "kernel": "prefill_gemm_kernel (gate/up + down grouped GEMMs of one call, tcgen05 fp16)",
            "achieved": gemm_tf,
            "peak": tflops,
            "unit": "TFLOP/s",
            "frac": (gemm_tf / tflops) if gemm_tf else None,
            "launch_us": gemm_ms * 1e3,
            "traffic": None,
            "peak_source": (f"{peak_kind} bf16_tflops (MEASURED_PEAKS.json); fp16 dense rate = bf16 "
                            "rate (nominal ratio 1:1)"),
            "per_unit": f"6 d f = {6 * D * F} FLOP per (token, expert) row; "
                        f"{T * K_TOP + T} rows per call",
        } if prefill else {
            "bound": "hbm",
            "kernel": kern_name,
            "achieved": kern_gbs,
            "peak": hbm,
            "unit": "GB/s",
            "frac": (kern_gbs / hbm) if kern_gbs else None,
            "launch_us": kern_ms / K * 1e3 if single else kern_ms / max(ncalls, 1) * 1e3,
            **({"launch_us_event_bracketed": bracketed_us,
                "launch_timing": "timed region / launches (one decode_kernel per step)"}
               if single else {}),
            "traffic": kernel_traffic(kern_bytes / K) if single else None,
            "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
                           else "fallback 6650 GB/s",
            "per_unit": per_unit,
        },
        "e2e": {"value": whole_job_rate(world, tok, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * D * 2, "d2h_bytes_per_step": T * D * 2},
        "gpu_launches": K * (1 if single else (8 if prefill else 6)),
        "clocks": clocks,
    }
    B.moe_destroy(ctx)
    return res, spec


def run_stack(args, world, rank, local):
    """48-layer stack: each step is one moe_forward_stack call (one CUDA graph
    of the 48 layers) on a new 32-token window."""
    import torch
    from sparse_moe_expert_gemv_b200 import binding as B
    from sparse_moe_expert_gemv_b200 import inputs as I

    spec = workload_spec(args)
    T, NL, SLOTS = spec["T"], 48, 4096
    K, W = args.steps, args.warmup
    ctx = B.moe_create(D, F, E, K_TOP, I.Q4)
    B.moe_configure(ctx, NL, 1, SLOTS, T)
    ranks = []
    for l in range(NL):
        bias, rank_of, _ = I.zipf_bias_np(args.seed, E, l)
        B.moe_set_router(ctx, l, I.router_np(args.seed, E, D, l), bias)
        for first in range(0, E, 64):
            c, s_, m = I.experts_torch(args.seed, I.Q4, D, F, l, first, 64, "cuda")
            B.moe_load_experts(ctx, l, first, 64, c, s_, m)
            del c, s_, m
        c, s_, m = I.shared_np(args.seed, I.Q4, D, F, l)
        B.moe_load_shared(ctx, l, c, s_, m)
        B.moe_set_norm(ctx, l, None, 1e-6)
        ranks.append(rank_of)
    B.moe_set_slots(ctx, I.slot_table_np(E, NL, SLOTS, np.stack(ranks)))
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    Be = B.moe_expert_bytes(D, F, I.Q4)

    n_win = K
    xs = np.stack([I.hidden_np(args.seed, T, D, window=i) for i in range(n_win)])
    x_host = torch.from_numpy(xs.view(np.int16)).pin_memory()
    x_dev0 = x_host.cuda()
    x_work = x_dev0.clone()
    # untimed pre-pass: per layer, the experts each step touches (from the
    # per-expert token counts of the call)
    scratch = x_dev0.clone()
    distinct = []
    for i in range(n_win):
        for l in range(NL):
            B.moe_forward(ctx, l, scratch[i], T)
            st = B.moe_get_stats(ctx)
            distinct.append(int((st["expert_count"] > 0).sum()))
    st0 = B.moe_get_stats(ctx)
    expert_bytes = float((np.array(distinct) + 1).sum() * Be)
    router_bytes = float(n_win * NL * E * D * 4)
    kern_bytes = expert_bytes + router_bytes
    # warm-up: every buffer's first call records its graph
    for i in range(n_win):
        B.moe_forward_stack(ctx, x_work[i], T)
    for _ in range(max(W - 1, 0)):
        B.moe_forward_stack(ctx, x_work[0], T)
    torch.cuda.synchronize()
    x_work.copy_(x_dev0)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(n_win):
            B.moe_forward_stack(ctx, x_work[i], T)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(world, ms)
    clocks = clk.summary()
    st1 = B.moe_get_stats(ctx)
    hits = st1["hits"] - st0["hits"]
    misses = st1["misses"] - st0["misses"]
    # end to end through the public call with host buffers
    out_host = torch.empty_like(x_host).pin_memory()
    xbuf = torch.empty((T, D), dtype=torch.int16, device="cuda")
    B.moe_forward_stack(ctx, xbuf, T)  # records the graph of this buffer
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for i in range(n_win):
        xbuf.copy_(x_host[i], non_blocking=True)
        B.moe_forward_stack(ctx, xbuf, T)
        out_host[i].copy_(xbuf, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, e0.elapsed_time(e1))
    B.moe_sync(ctx, 60000)
    hbm, _, peak_kind = peaks()
    gbs = kern_bytes / (ms_max * 1e-3) / 1e9
    single = T <= 32
    res = {
        "metric": "stack MoE tokens/s", "value": whole_job_rate(world, T * K, ms_max), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms_max / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "q4-g32 weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded generator; random-init weights of the stack's shape)",
        "config": {"workload": spec["name"], "tokens_per_step": T, "layers": NL,
                   "l2": "no flush: one step reads ~48 x 100+ MB of experts (>> 126 MB L2)",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "timing": "K moe_forward_stack calls (each one CUDA graph), CUDA events"},
        "expert_weight_gbs": expert_bytes / (ms_max * 1e-3) / 1e9,
        "distinct_experts_per_layer": float(np.mean(distinct)),
        "slot_hit_rate": hits / max(hits + misses, 1),
        "roofline": {"bound": "hbm",
                     "kernel": ("decode_kernel x 48 (one launch per layer)" if single else
                                "multi-launch layer path x 48"),
                     "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "traffic": None,
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)",
                     "per_unit": f"{Be} B per touched expert per layer (shared included) + "
                                 f"{E * D * 4} B router W per layer"},
        "e2e": {"value": whole_job_rate(world, T * K, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * D * 2, "d2h_bytes_per_step": T * D * 2},
        "gpu_launches": K * NL * (1 if single else 6),
        "clocks": clocks,
    }
    B.moe_destroy(ctx)
    return res, spec


def cpu_baseline(args, spec, seconds):
    """The oracle, as it stands, on a bounded sample of the same workload."""
    import oracle as O
    from sparse_moe_expert_gemv_b200 import inputs as I
    O.build()
    T = spec["T"]
    W = I.router_np(args.seed, E, D, 0)
    bias = I.zipf_bias_np(args.seed, E, 0)[0] if spec["zipf"] else None
    cache = {}
    tok = 0
    t0 = time.perf_counter()
    win = 0
    while time.perf_counter() - t0 < seconds:
        x = I.hidden_np(args.seed, min(T, 4), D, window=100000 + win)
        win += 1
        lg = O.router(x, W, bias)
        idx, _, _ = O.topk(lg, K_TOP)
        experts = {}
        for e in set(idx.reshape(-1).tolist()):
            if e not in cache:
                cache[e] = I.expert_np(args.seed, spec["fmt"], D, F, 0, e)
            experts[e] = cache[e]
        O.moe_layer(x, fmt=spec["fmt"], d=D, f=F, E=E, k=K_TOP, router_w=W, router_bias=bias,
                    experts=experts, shared=I.shared_np(args.seed, spec["fmt"], D, F, 0))
        tok += x.shape[0]
        if len(cache) > 256:
            cache.clear()
    dt = time.perf_counter() - t0
    return {"value": tok / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{win} windows of {min(T, 4)} tokens through the full layer "
                      f"(fp64 scalar C, single thread, {dt:.1f} s)"}


def run_reference(args):
    """Reference arm: the oracle (scalar fp64 C) on the host cores."""
    spec = workload_spec(args)
    import oracle as O
    from sparse_moe_expert_gemv_b200 import inputs as I
    O.build()
    W = I.router_np(args.seed, E, D, 0)
    bias = I.zipf_bias_np(args.seed, E, 0)[0] if spec["zipf"] else None
    shared = I.shared_np(args.seed, spec["fmt"], D, F, 0)

    def step(i):
        x = I.hidden_np(args.seed, 1, D, window=200000 + i)
        lg = O.router(x, W, bias)
        idx, _, _ = O.topk(lg, K_TOP)
        experts = {e: I.expert_np(args.seed, spec["fmt"], D, F, 0, e)
                   for e in set(idx.reshape(-1).tolist())}
        O.moe_layer(x, fmt=spec["fmt"], d=D, f=F, E=E, k=K_TOP, router_w=W, router_bias=bias,
                    experts=experts, shared=shared)
        return 1

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    tok = sum(step(args.warmup + i) for i in range(args.steps))
    dt = time.perf_counter() - t0
    v = tok / dt
    return {"impl": "reference", "metric": "decode MoE tokens/s" if args.workload != "prefill"
            else "prefill MoE tokens/s", "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec["name"],
                       "sample": "each step: 1 token through the full layer"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": "1 token per step through the full layer (router over "
                                       "512 experts, its 10 experts + shared, fp64)"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    world, rank, local = dist_setup(args)
    from sparse_moe_expert_gemv_b200 import build as _b
    _b.build()
    if args.workload == "stack":
        res, spec = run_stack(args, world, rank, local)
    else:
        res, spec = run_native(args, world, rank, local)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args, spec, args.cpu_seconds)
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
