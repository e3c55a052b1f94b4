#!/usr/bin/env python
"""Benchmark of the sparse MoE expert layer on B200.

Headline workload: one Flash-Next-shaped MoE layer in decode, d=2048,
f=768, E=512, top-10 renormalised softmax + 1 shared expert, 4-bit symmetric
group-32 experts, bf16 hidden N(0,1), verify window T=4, uniform routing.  A
step = one moe_forward call (router, top-k, residency lookup, bucketing,
dequant-SwiGLU experts, combine + residual) on a new 4-token window.  Steps
rotate over --rot-layers independent copies of the layer's weights (16 x
1.36 GB by default), so the weights a step reads were evicted from the 126
MB L2 long before (no flush needed).

At one GPU the same JSON line also carries the other workloads of the
metric, each with its own roofline, end-to-end figure and clocks:
  "prefill"  an 8192-token chunk through one layer (Q4, Zipf(1.1) routing):
             prefill MoE tokens/s, tensor-pipe roofline of its grouped GEMMs;
  "q2"       2-bit asymmetric g64 experts, Zipf(1.1) routing, 64 sequences x
             T tokens per call, T = 1..5: tokens/s and expert GB/s per T;
  "stack"    the 48-layer stack (RMSNorm -> router -> experts -> combine per
             layer, 4096-slot residency table), 32 tokens per step.
(--no-extras drops them; --workload q2|prefill|stack makes one of them the
headline instead.)  --workload tier runs the host tier: 4 layers whose
experts are backed in pinned host memory, a 512-slot HBM cache, Zipf-routed
16-token windows through moe_forward_tiered, both replacement policies and
the all-HBM forward of the same windows (use it with --no-cpu-baseline).

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
    ap.add_argument("--workload", default="decode", choices=["decode", "q2", "prefill", "stack", "tier", "ep"])
    ap.add_argument("--T", type=int, default=4, help="window (decode) / per-sequence window (q2)")
    ap.add_argument("--rot-layers", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-extras", action="store_true",
                    help="headline only (no prefill / q2 / stack objects)")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--experts", type=int, default=512,
                    help="routed experts per layer (256: the pruned configuration)")
    a = ap.parse_args()
    if a.steps is None:
        a.steps = {"prefill": 20, "stack": 10, "tier": 100, "ep": 10}.get(a.workload, 200)
    return a


# ----------------------------------------------------------------- helpers
def _traffic_record(name):
    """A committed ncu traffic record (profiles/<name>), or None when it is
    missing or the kernel sources changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", name)
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
    return rec


def kernel_traffic(kernel_bytes_per_launch):
    """Per-launch DRAM traffic of decode_kernel from the committed ncu record,
    scaled to this run's algorithmic bytes per launch (the record's launch
    routed a different window)."""
    rec = _traffic_record("decode_kernel_traffic.json")
    return None if rec is None else rec["traffic_over_algorithmic"] * kernel_bytes_per_launch


def q2_traffic(bytes_per_call):
    """DRAM bytes of the four expert launches of one Q2 call (GEMM and GEMV,
    gate/up and down) from the committed ncu record, scaled to this run's
    algorithmic expert bytes per call."""
    rec = _traffic_record("q2_experts_traffic.json")
    return None if rec is None else rec["traffic_over_algorithmic"] * bytes_per_call


def prefill_traffic(flops_per_call):
    """DRAM bytes of the two grouped-GEMM launches of one 8192-token chunk,
    from the committed ncu record (scaled by FLOPs when this chunk's work
    differs from the record's)."""
    rec = _traffic_record("prefill_gemm_traffic.json")
    if rec is None:
        return None
    return rec["bytes_per_call"] * flops_per_call / rec["flops_per_call"]


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, kind): the measured copy bandwidth and
    cuBLAS bf16 rate in MEASURED_PEAKS.json when the file is present, else an
    earlier measurement of the same part (kind "fallback")."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def peak_source(kind, what):
    """What a roofline's peak is: `what` is "hbm" or "tensor"."""
    if kind == "measured":
        return ("measured hbm_gbs (MEASURED_PEAKS.json)" if what == "hbm" else
                "measured bf16_tflops burst (MEASURED_PEAKS.json); fp16 dense rate = bf16 rate "
                "(nominal ratio 1:1)")
    return ("fallback 6650 GB/s (no MEASURED_PEAKS.json)" if what == "hbm" else
            "fallback 1590 TFLOP/s bf16 burst (no MEASURED_PEAKS.json); fp16 dense rate = bf16 rate "
            "(nominal ratio 1:1)")


def host_info():
    """Logical cores and CPU model of this host (for the CPU baselines)."""
    model = None
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count() or 1
    return {"nproc": os.cpu_count(), "usable_cores": usable, "cpu_model": model}


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
def workload_spec(name, T=4):
    from sparse_moe_expert_gemv_b200 import inputs as I
    if name == "decode":
        return dict(kind=name, name=f"one MoE layer decode, d=2048 f=768 E={E} top-10 + shared, "
                                    f"Q4 g32, T={T}, uniform routing",
                    fmt=I.Q4, zipf=False, T=T, seqs=1, prefill=False, metric="decode MoE tokens/s")
    if name == "q2":
        return dict(kind=name, name=f"one MoE layer decode, Q2 g64 asym, Zipf(1.1) routing, "
                                    f"64 sequences x T={T}",
                    fmt=I.Q2, zipf=True, T=T * 64, seqs=64, prefill=False, metric="decode MoE tokens/s")
    if name == "stack":
        return dict(kind=name, name="48-layer MoE stack (RMSNorm -> router -> experts -> combine + "
                                    f"residual), d=2048 f=768 E={E} top-10 + shared, Q4 g32, "
                                    "4096-slot residency table by Zipf rank, Zipf(1.1) routing, "
                                    "T=4 x batch 8 = 32 tokens",
                    fmt=I.Q4, zipf=True, T=32, seqs=8, prefill=False, metric="stack MoE tokens/s")
    return dict(kind="prefill", name=f"prefill chunk, 8192 tokens, one MoE layer, d=2048 f=768 E={E} "
                                     "top-10 + shared, Q4 g32, Zipf(1.1) routing",
                fmt=I.Q4, zipf=True, T=8192, seqs=1, prefill=True, metric="prefill MoE tokens/s")


def build_native(args, spec, n_rot, max_tokens=None):
    import torch
    from sparse_moe_expert_gemv_b200 import binding as B
    from sparse_moe_expert_gemv_b200 import inputs as I
    ctx = B.moe_create(D, F, E, K_TOP, spec["fmt"])
    B.moe_configure(ctx, n_rot, 1, 0, max_tokens or spec["T"])
    for l in range(n_rot):
        W = I.router_np(args.seed, E, D, l)
        bias = I.zipf_bias_np(args.seed, E, l)[0] if spec["zipf"] else None
        B.moe_set_router(ctx, l, W, bias)
        for first in range(0, E, 64):
            c, s, m = I.experts_torch(args.seed, spec["fmt"], D, F, l, first, 64, "cuda")
            B.moe_load_experts(ctx, l, first, 64, c, s, m)
            del c, s, m
        c, s, m = I.experts_torch(args.seed, spec["fmt"], D, F, l, I.SHARED_INDEX, 1, "cuda")
        B.moe_load_shared(ctx, l, c, s, m)
        del c, s, m
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return ctx


def run_native(args, world, spec, n_rot, K, W):
    """Build the layer copies, measure, free."""
    from sparse_moe_expert_gemv_b200 import binding as B
    ctx = build_native(args, spec, n_rot)
    try:
        return measure(args, world, ctx, spec, n_rot, K, W)
    finally:
        B.moe_destroy(ctx)


def measure(args, world, ctx, spec, n_rot, K, W):
    """K timed steps of one workload on a built context (n_rot layer copies)."""
    import torch
    from sparse_moe_expert_gemv_b200 import binding as B
    from sparse_moe_expert_gemv_b200 import inputs as I

    T = spec["T"]
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
    prefill = spec["prefill"]
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
        kern_name = ("the experts of one call: prefill_gemm_kernel (gate/up + down, experts with "
                     ">= 24 tokens) + expert_gemv_kernel (gate/up + down, the other experts, beside the GEMM)")
        per_unit = f"{Be} B per touched expert (codes+scales), shared expert included"
    kern_gbs = kern_bytes / (kern_ms * 1e-3) / 1e9 if kern_ms > 0 else None
    res = {
        "metric": spec["metric"],
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
                                 "combine": comb_ms / max(ncalls, 1),
                                 "timing": "a second, event-bracketed pass of the same steps"},
        "roofline": {
            "bound": "tensor",
            "kernel": ("the experts of one call: prefill_gemm_kernel (gate/up + down grouped GEMMs, "
                       "tcgen05 fp16, experts with >= 24 tokens) + expert_gemv_kernel (the other "
                       "experts)"),
            "achieved": gemm_tf,
            "peak": tflops,
            "unit": "TFLOP/s",
            "frac": (gemm_tf / tflops) if gemm_tf else None,
            "launch_us": gemm_ms * 1e3,
            "traffic": None,
            "peak_source": peak_source(peak_kind, "tensor"),
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
            "traffic": (kernel_traffic(kern_bytes / K) if single else
                        q2_traffic(kern_bytes / K) if spec["kind"] == "q2" and spec["T"] == 256 else None),
            "peak_source": peak_source(peak_kind, "hbm"),
            "per_unit": per_unit,
        },
        "e2e": {"value": whole_job_rate(world, tok, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * D * 2, "d2h_bytes_per_step": T * D * 2},
        # chunks: router, top-k, column scan, scan, scatter, 2 GEMMs, 2 GEMVs,
        # combine, and one more: the split router's sum (the Q2 chunks of 64-320
        # tokens) or the column scan's counting pass (8192 tokens)
        "gpu_launches": K * (1 if single else 11),
        "clocks": clocks,
    }
    if single:
        # one launch per step: the profile pass only brackets that launch
        del res["segments_ms_per_step"]
    if prefill:
        res["roofline"]["traffic"] = prefill_traffic(flops)
    return res


def run_stack(args, world, K, W):
    """48-layer stack: each step is one moe_forward_stack call (one CUDA graph
    of the 48 layers) on a new 32-token window."""
    import torch
    from sparse_moe_expert_gemv_b200 import binding as B
    from sparse_moe_expert_gemv_b200 import inputs as I

    spec = workload_spec("stack")
    T, NL, SLOTS = spec["T"], 48, 4096
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
        c, s_, m = I.experts_torch(args.seed, I.Q4, D, F, l, I.SHARED_INDEX, 1, "cuda")
        B.moe_load_shared(ctx, l, c, s_, m)
        del c, s_, m
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
                     "peak_source": peak_source(peak_kind, "hbm"),
                     "per_unit": f"{Be} B per touched expert per layer (shared included) + "
                                 f"{E * D * 4} B router W per layer"},
        "e2e": {"value": whole_job_rate(world, T * K, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * D * 2, "d2h_bytes_per_step": T * D * 2},
        "gpu_launches": K * NL * (1 if single else 6),
        "clocks": clocks,
    }
    B.moe_destroy(ctx)
    return res


# ------------------------------------------------ the oracle on host cores
def oracle_rows_threaded(x_rows, spec, W, bias, experts, shared, threads, norm=False):
    """The oracle's layer on token rows, the rows split over `threads`
    host threads (tokens are independent; the C oracle runs without the
    GIL).  `experts` maps id -> packed bytes for every id a row selects."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle as O

    chunks = [c for c in np.array_split(np.arange(x_rows.shape[0]), threads) if c.size]

    def one(c):
        x = np.ascontiguousarray(x_rows[c])
        h = O.rmsnorm(x, None, 1e-6) if norm else x
        idx, _, _ = O.topk(O.router(h, W, bias), K_TOP)
        need = {e: experts[e] for e in set(idx.reshape(-1).tolist())}
        O.moe_layer(x, fmt=spec["fmt"], d=D, f=F, E=E, k=K_TOP, router_w=W, router_bias=bias,
                    experts=need, shared=shared, norm=norm)
        return c.size

    with ThreadPoolExecutor(len(chunks)) as ex:
        return sum(ex.map(one, chunks))


def host_experts(args, fmt, layer, on_gpu):
    """Packed bytes of every expert (and the shared one) of one layer, made
    before any timing: on the GPU with the torch generator when there is one,
    else with the numpy generator on host threads."""
    from concurrent.futures import ThreadPoolExecutor

    from sparse_moe_expert_gemv_b200 import inputs as I
    out = {}
    if on_gpu:
        for first in range(0, E, 64):
            c, s, m = I.experts_torch(args.seed, fmt, D, F, layer, first, 64, "cuda")
            c, s = c.cpu().numpy(), s.cpu().numpy().view(np.uint16)
            m = None if m is None else m.cpu().numpy().view(np.uint16)
            for i in range(64):
                out[first + i] = (c[i], s[i], None if m is None else m[i])
        c, s, m = I.experts_torch(args.seed, fmt, D, F, layer, I.SHARED_INDEX, 1, "cuda")
        shared = (c[0].cpu().numpy(), s[0].cpu().numpy().view(np.uint16),
                  None if m is None else m[0].cpu().numpy().view(np.uint16))
        return out, shared
    with ThreadPoolExecutor(host_info()["usable_cores"]) as ex:
        vals = list(ex.map(lambda e: I.expert_np(args.seed, fmt, D, F, layer, e), range(E)))
    return dict(enumerate(vals)), I.shared_np(args.seed, fmt, D, F, layer)


def cpu_baseline(args, spec, seconds, on_gpu=True, norm=False, tokens=None, layers_per_token=1):
    """The oracle, as it stands, on a bounded sample of the same workload:
    token windows of the workload through the full layer, each window's
    tokens split over the host's cores.  Runs for about `seconds`."""
    from sparse_moe_expert_gemv_b200 import inputs as I
    import oracle as O
    O.build()
    info = host_info()
    threads = info["usable_cores"]
    W = I.router_np(args.seed, E, D, 0)
    bias = I.zipf_bias_np(args.seed, E, 0)[0] if spec["zipf"] else None
    experts, shared = host_experts(args, spec["fmt"], 0, on_gpu)
    per = tokens or min(spec["T"], max(threads, 4))
    tok, win = 0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        x = I.hidden_np(args.seed, per, D, window=100000 + win)
        tok += oracle_rows_threaded(x, spec, W, bias, experts, shared, threads, norm=norm)
        win += 1
    dt = time.perf_counter() - t0
    value = tok / dt / layers_per_token
    what = (f"{win} windows of {per} tokens through one full layer"
            + (f" (a token of the stack passes {layers_per_token} layers: tokens/s = "
               f"layer-tokens/s / {layers_per_token})" if layers_per_token > 1 else ""))
    return {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{what}; fp64 scalar C, each window's tokens split over {threads} "
                      f"host threads; {dt:.1f} s", **info}


def run_tier(args, world, K, W):
    """Host tier: the experts' backing copies in pinned host memory, a slot
    pool of a quarter of the (layer, expert) pairs in HBM, Zipf-routed
    windows through moe_forward_tiered (route, bring the misses in, forward);
    both replacement policies, and the all-HBM forward of the same windows for
    comparison.  Timed with CUDA events around the K windows (the miss path
    synchronises the stream once per window to read the routing back)."""
    import torch
    from sparse_moe_expert_gemv_b200 import binding as B
    from sparse_moe_expert_gemv_b200 import inputs as I
    NL, T, slots = 4, 16, 512
    xs = torch.from_numpy(np.stack([I.hidden_np(args.seed, T, D, window=i) for i in range(W + K)])
                          .view(np.int16)).cuda()

    def build(tier, policy):
        ctx = B.moe_create(D, F, E, K_TOP, I.Q4)
        if tier:
            B.moe_set_host_tier(ctx, 1, policy, 64.0)
        B.moe_configure(ctx, NL, 1, slots if tier else 0, T)
        for l in range(NL):
            B.moe_set_router(ctx, l, I.router_np(args.seed, E, D, l), I.zipf_bias_np(args.seed, E, l)[0])
            for first in range(0, E, 64):
                c, s_, m = I.experts_torch(args.seed, I.Q4, D, F, l, first, 64, "cuda")
                B.moe_load_experts(ctx, l, first, 64, c, s_, m)
                del c, s_, m
            c, s_, m = I.experts_torch(args.seed, I.Q4, D, F, l, I.SHARED_INDEX, 1, "cuda")
            B.moe_load_shared(ctx, l, c, s_, m)
        torch.cuda.synchronize()
        return ctx

    def run(ctx, fwd):
        work = xs.clone()
        for i in range(W):
            fwd(ctx, i % NL, work[i], T)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        st0 = B.moe_tier_stats(ctx) if fwd is B.moe_forward_tiered else None
        e0.record()
        for i in range(W, W + K):
            fwd(ctx, i % NL, work[i], T)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        st1 = B.moe_tier_stats(ctx) if st0 else None
        B.moe_sync(ctx, 60000)
        return ms, (None if st0 is None else {k: st1[k] - st0[k] for k in st1})

    out = {}
    ctx = build(False, 0)
    ms_hbm, _ = run(ctx, B.moe_forward)
    B.moe_destroy(ctx)
    for name, pol in (("lru", B.TIER_LRU), ("adaptive", B.TIER_ADAPTIVE)):
        ctx = build(True, pol)
        ms, d = run(ctx, B.moe_forward_tiered)
        B.moe_destroy(ctx)
        torch.cuda.empty_cache()
        req = d["hits"] + d["misses"]
        out[name] = {"value": K * T / (ms * 1e-3), "unit": "tokens/s", "ms_per_window": ms / K,
                     "hit_rate": d["hits"] / max(req, 1), "misses_per_window": d["misses"] / K,
                     "h2d_gbs": d["bytes"] / (ms * 1e-3) / 1e9}
    return {"metric": "tier MoE tokens/s", "value": out["adaptive"]["value"], "unit": "tokens/s",
            "n_gpus": 1, "steps": K, "warmup": W, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "q4-g32 weights, bf16 activations, fp32 accumulate",
            "data": "synthetic (seeded generator; random-init weights of the layer's shape)",
            "config": {"workload": f"{NL} MoE layers, d=2048 f=768 E={E} top-10 + shared, Q4 g32, Zipf(1.1) "
                                   f"routing, windows of T={T}; experts backed in pinned host memory, "
                                   f"{slots} HBM slots ({slots / (NL * E):.0%} of the pairs)",
                       "tokens_per_step": T, "parallelism": "1 GPU",
                       "timing": "CUDA events around K moe_forward_tiered calls (each reads its routing back)"},
            "policies": out,
            "all_hbm": {"value": K * T / (ms_hbm * 1e-3), "unit": "tokens/s", "ms_per_window": ms_hbm / K},
            "gpu_launches": None}


def ep_launches_per_step(N, rows, max_rows):
    """Library kernels one ExpertParallelMoE.forward launches for N tokens of
    its own and `rows` received rows (8192-token chunks: the tensor-core
    router needs no split).  A chunk step on n rows adds a column-count pass
    when its column scan is split (n / 8 mask blocks over ranges of 64)."""
    def colcount(n):
        return 1 if min(32, (n + 7) // 8 // 64) > 1 else 0
    route = 5 + colcount(N)                       # router, top-k, [count], column scan, scan, scatter
    dispatch = 3                                  # count, offsets, place + copy
    given = 0
    for a in range(0, rows, max_rows):            # mask, [count], column scan, scan, scatter,
        given += 9 + colcount(min(max_rows, rows - a))   # two GEMM, two GEMV, combine
    shared = 9 + colcount(N)
    return route + dispatch + given + shared + 1  # + the combine


def run_ep(args, world, rank, K, W):
    """Expert parallelism (ep.py): each rank holds E / world experts of the
    layer (router and shared expert replicated) and 8192 tokens of its own;
    one step is ExpertParallelMoE.forward on them (route, dispatch by owner,
    NCCL all-to-all, owners' experts, all-to-all back, shared expert,
    combine).  With one GPU the process group has one rank and the
    exchange is a local copy; the one-GPU layer (moe_prefill) on the same
    tokens is timed beside it.  Phases are timed in one extra untimed step."""
    import socket

    import torch
    import torch.distributed as dist
    from sparse_moe_expert_gemv_b200 import binding as B
    from sparse_moe_expert_gemv_b200 import inputs as I
    from sparse_moe_expert_gemv_b200.ep import DeviceOps, Exchange, ExpertParallelMoE

    own_group = not dist.is_initialized()
    if own_group:
        with socket.socket() as s_:
            s_.bind(("127.0.0.1", 0))
            port = s_.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                device_id=torch.device("cuda", 0))
    N = 8192
    per = E // world
    ctx = B.moe_create(D, F, E, K_TOP, I.Q4)
    try:
        B.moe_configure(ctx, 1, 1, 0, N * K_TOP)
        B.moe_set_router(ctx, 0, I.router_np(args.seed, E, D, 0), I.zipf_bias_np(args.seed, E, 0)[0])
        for first in range(rank * per, (rank + 1) * per, 64):
            n = min(64, (rank + 1) * per - first)
            c, s_, m = I.experts_torch(args.seed, I.Q4, D, F, 0, first, n, "cuda")
            B.moe_load_experts(ctx, 0, first, n, c, s_, m)
            del c, s_, m
        c, s_, m = I.experts_torch(args.seed, I.Q4, D, F, 0, I.SHARED_INDEX, 1, "cuda")
        B.moe_load_shared(ctx, 0, c, s_, m)
        del c, s_, m
        torch.cuda.synchronize()
        ops = DeviceOps(B, ctx, d=D, k=K_TOP, E=E, max_tokens=N * K_TOP, has_shared=True)
        marks = []
        moe = ExpertParallelMoE(ops, Exchange(), on_phase=None)
        x0 = torch.from_numpy(I.hidden_np(args.seed, N, D, window=1000 + rank).view(np.int16)).cuda()
        x = x0.clone()
        for _ in range(W):
            x.copy_(x0)
            moe.forward(0, x, N)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) as cs:
            e0.record()
            for _ in range(K):
                x.copy_(x0)
                moe.forward(0, x, N)
            e1.record()
            torch.cuda.synchronize()
        barrier(world)
        ms_max = max_over_ranks(world, e0.elapsed_time(e1))
        clocks = cs.summary()
        # phases of one more step
        ev0 = torch.cuda.Event(enable_timing=True)

        def on_phase(name):
            ev = torch.cuda.Event(enable_timing=True)
            ev.record()
            marks.append((name, ev))

        moe.on_phase = on_phase
        x.copy_(x0)
        ev0.record()
        moe.forward(0, x, N)
        torch.cuda.synchronize()
        moe.on_phase = None
        seg, prev = {}, ev0
        for name, ev in marks:
            seg[name] = prev.elapsed_time(ev)
            prev = ev
        # end to end: the input copied in from pinned host memory and the
        # result read back, every step, through the same public call
        x_host = x0.cpu().pin_memory()
        out_host = torch.empty_like(x_host).pin_memory()
        barrier(world)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(K):
            x.copy_(x_host, non_blocking=True)
            moe.forward(0, x, N)
            out_host.copy_(x, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(world, e0.elapsed_time(e1))
        one_gpu = None
        if world == 1:   # the one-GPU layer on the same tokens, for comparison
            for _ in range(W):
                x.copy_(x0)
                B.moe_prefill(ctx, 0, x, N)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(K):
                x.copy_(x0)
                B.moe_prefill(ctx, 0, x, N)
            e1.record()
            torch.cuda.synchronize()
            one_gpu = {"ms_per_step": e0.elapsed_time(e1) / K,
                       "value": K * N / (e0.elapsed_time(e1) * 1e-3), "unit": "tokens/s"}
        B.moe_sync(ctx, 120000)
    finally:
        B.moe_destroy(ctx)
    _, tflops_peak, peak_kind = peaks()
    flops = 6.0 * D * F * (N * K_TOP + N)
    t_exp = (seg["experts"] + seg["shared"]) * 1e-3
    P = N * K_TOP
    gather_bytes = N * D * 2 + P * D * 2
    combine_bytes = P * D * 2 + N * D * 4 + 2 * N * D * 2 + P * 8   # fp16 y rows, fp32 shared, x
    res = {
        "metric": "expert-parallel MoE tokens/s", "value": whole_job_rate(world, N * K, ms_max),
        "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms_max / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "q4-g32 weights, bf16 activations, fp16 tensor-core operands, fp32 accumulate",
        "data": "synthetic (seeded generator; random-init weights of the layer's shape)",
        "config": {"workload": f"expert-parallel MoE layer, d=2048 f=768 E={E} top-10 + shared, Q4 g32, "
                               f"Zipf(1.1) routing, {N} tokens per rank, {per} experts per rank",
                   "tokens_per_step": N * world, "parallelism": f"ep{world}",
                   "l2": "no flush: a step moves ~1 GB of rows and outputs (>> 126 MB L2)",
                   "timing": "K ExpertParallelMoE.forward calls, CUDA events, max over ranks"},
        "segments_ms_one_step": seg,
        "roofline": {"bound": "tensor", "kernel": "owners' experts + shared expert (moe_experts_given)",
                     "achieved": flops / t_exp / 1e12, "peak": tflops_peak, "unit": "TFLOP/s",
                     "frac": flops / t_exp / 1e12 / tflops_peak, "traffic": None,
                     "peak_source": peak_source(peak_kind, "bf16"),
                     "per_unit": "6 d f FLOP per (token, expert) row; the rank's 8192 x (10 + 1) rows"},
        "dispatch_gbs": gather_bytes / (seg["dispatch"] * 1e-3) / 1e9,
        "combine_gbs": combine_bytes / (seg["combine"] * 1e-3) / 1e9,
        "e2e": {"value": whole_job_rate(world, N * K, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": N * D * 2, "d2h_bytes_per_step": N * D * 2},
        "gpu_launches": K * ep_launches_per_step(N, ops.last_rows, N * K_TOP),
        "clocks": clocks,
    }
    if one_gpu:
        res["one_gpu_layer"] = one_gpu
    if own_group:
        dist.destroy_process_group()
    return res


def run_reference(args):
    """Reference arm: the oracle (scalar fp64 C) on the host cores, on the
    headline's workload: each step is one window of the workload's tokens
    through the full layer (capped at 8 tokens for the prefill and stack
    workloads, whose steps the oracle cannot finish in minutes)."""
    spec = workload_spec(args.workload, args.T)
    import oracle as O
    from sparse_moe_expert_gemv_b200 import inputs as I
    O.build()
    info = host_info()
    threads = info["usable_cores"]
    W = I.router_np(args.seed, E, D, 0)
    bias = I.zipf_bias_np(args.seed, E, 0)[0] if spec["zipf"] else None
    experts, shared = host_experts(args, spec["fmt"], 0, on_gpu=False)
    per = spec["T"] if spec["kind"] in ("decode", "q2") and spec["T"] <= 8 else 8
    norm = spec["kind"] == "stack"

    def step(i):
        x = I.hidden_np(args.seed, per, D, window=i)
        return oracle_rows_threaded(x, spec, W, bias, experts, shared, threads, norm=norm)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    tok = sum(step(args.warmup + i) for i in range(args.steps))
    dt = time.perf_counter() - t0
    v = tok / dt / (48 if spec["kind"] == "stack" else 1)
    same = per == spec["T"]
    sample = (f"each step: {per} tokens (window {'= the workload' if same else 'sample'}) through "
              f"the full layer{' (x 48 layers for the stack rate)' if norm else ''}, fp64 scalar C, "
              f"tokens split over {threads} host threads")
    return {"impl": "reference", "metric": spec["metric"], "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec["name"], "tokens_per_step": per, "same_window": same},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample, **info},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def q2_sweep(args, world, K, W):
    """Config Q2: one Q2 context (4 rotated layer copies), T = 1..5 tokens per
    sequence x 64 sequences per call."""
    from sparse_moe_expert_gemv_b200 import binding as B
    spec0 = workload_spec("q2", 5)
    n_rot = 4
    ctx = build_native(args, spec0, n_rot, max_tokens=spec0["T"])
    out = {}
    try:
        for T in range(1, 6):
            r = measure(args, world, ctx, workload_spec("q2", T), n_rot, K, W)
            out[f"T{T}"] = {key: r[key] for key in
                            ("value", "unit", "ms_per_step", "steps", "warmup", "expert_weight_gbs",
                             "distinct_experts_per_step", "roofline", "e2e", "gpu_launches",
                             "segments_ms_per_step", "clocks")}
            out[f"T{T}"]["tokens_per_step"] = 64 * T
    finally:
        B.moe_destroy(ctx)
    return {"workload": "one MoE layer decode, d=2048 f=768 E=512 top-10 + shared, Q2 g64 asym "
                        "(fp16 scale + min), Zipf(1.1) routing, 64 sequences x T tokens per call",
            "metric": "decode MoE tokens/s", "by_T": out}


def main():
    global E
    args = parse()
    E = args.experts
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    world, rank, local = dist_setup(args)
    from sparse_moe_expert_gemv_b200 import build as _b
    _b.build()
    spec = workload_spec(args.workload, args.T)
    if args.workload == "stack":
        res = run_stack(args, world, args.steps, args.warmup)
    elif args.workload == "tier":
        res = run_tier(args, world, args.steps, args.warmup)
    elif args.workload == "ep":
        res = run_ep(args, world, rank, args.steps, args.warmup)
    else:
        n_rot = args.rot_layers if args.workload == "decode" else min(args.rot_layers, 4)
        res = run_native(args, world, spec, n_rot, args.steps, args.warmup)
    extras = world == 1 and not args.no_extras and args.workload == "decode" and E == 512
    if extras:
        ks, ws = args.extra_steps, 3
        pre = run_native(args, world, workload_spec("prefill"), 2, ks, ws)
        if not args.no_cpu_baseline:
            pre["cpu_baseline"] = cpu_baseline(args, workload_spec("prefill"), args.cpu_seconds,
                                               tokens=16)
        res["prefill"] = pre
        res["q2"] = q2_sweep(args, world, 2 * ks, ws)
        st = run_stack(args, world, max(ks // 2, 3), ws)
        if not args.no_cpu_baseline:
            st["cpu_baseline"] = cpu_baseline(args, workload_spec("stack"), args.cpu_seconds,
                                              norm=True, tokens=8, layers_per_token=48)
        res["stack"] = st
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
