"""Benchmark: Ring Attention blockwise exact attention, forward + backward.

One step = the whole hot path on one batch of synthetic inputs: ring_attention
forward (O, LSE) then backward (dQ, dK, dV recomputed from the saved LSE),
for the 128K-token causal workload (B=1, H=32, D=128, S=131072, P=8 virtual
ring ranks, chunks of 512, causal_block_size=1, bf16 N(0,1) inputs).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--mode fwdbwd|fwd|step] [--ring]
                    [--no-e2e] [--no-cpu-baseline]

--mode fwd times the forward alone; --mode step times the forward as the
pages' ring runs it on one GPU: P virtual ranks x P per-step calls (ra_step,
the tensor-core kernel in ring-step mode, each merging into its rank's fp32
running state in HBM) plus ra_finalize per rank.

Multi-GPU (torchrun, one process per GPU): by default every rank runs an
independent replica of the workload; the value is all ranks' work divided by
the slowest rank's device time ("scaling": "weak").  With --ring the
sequence is sharded over the ranks instead and key/value blocks travel round
the ring over NCCL (forward; "scaling": "strong").

Prints ONE JSON line on rank 0.  TFLOP/s counts only algorithmic work:
4*D per visible (query, key) pair for the forward, 10*D for the backward.
Besides the device-timed value it carries: "e2e", the same step through the
host-buffer API (HostStep -> ra_train_step_host, pinned H2D / D2H copies
inside the timed region); "roofline" for the backward kernel (measured peaks,
DRAM bytes per launch from the committed full-size ncu capture); "mufu", the
measured MUFU ex2 rate (the forward's second ceiling); "clocks" sampled during
the timed region; and "cpu_baseline", the float64 oracle on a bounded sample.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s (fwd, fwd+bwd) at 32K-1M tokens; % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The backward kernel's sources; the committed DRAM capture is void once any of them changes.
KERNEL_SRCS = [os.path.join(ROOT, "long_context_exact_ordered_b200", "csrc", f)
               for f in ("ra_bwd_sm100.cuh", "ra_common.cuh", "ptx.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ra_bwd_sm100_causal128k_dram.md")


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(world, backend):
    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def aggregate(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / seconds_max if seconds_max > 0 else 0.0


# ---------------------------------------------------------------- measured peaks / clocks

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.uuid = gpu_uuid
        self.proc = None
        self.out = os.path.join("/tmp", f"ra_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.out, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in open(self.out):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) >= 8:
                rows.append(parts)
        os.unlink(self.out)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v.lower() == "active"})
        power = [float(r[2]) for r in rows if re.match(r"^[0-9.]+$", r[2])]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(power) if power else None}


def mufu_rate(dev):
    """ex2 per clock per SM from the debug build's microbenchmark (None if that build is absent)."""
    import torch

    try:
        from long_context_exact_ordered_b200 import _lib

        dbg = _lib.load_count()
    except (ImportError, OSError, AttributeError):
        return None
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device=dev)
    sink = torch.zeros(512, dtype=torch.float32, device=dev)
    iters = 4096
    s = torch.cuda.current_stream(dev).cuda_stream
    for _ in range(2):
        if dbg.ra_debug_ex2_rate(iters, sms, cycles.data_ptr(), sink.data_ptr(), s) != 0:
            return None
    torch.cuda.synchronize(dev)
    return 512 * 8 * iters / cycles.double().mean().item(), sms


def kernel_sources_sha256() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SRCS:
        h.update(open(f, "rb").read())
    return h.hexdigest()


def traffic_per_launch():
    """dram bytes per launch of the backward kernel from the committed ncu summary,
    or None when the kernel source changed since those counters were taken."""
    try:
        text = open(TRAFFIC_FILE).read()
    except OSError:
        return None, None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"kernel_sources_sha256:\s*([0-9a-f]+)", text)
    if not m or not s:
        return None, None
    cur = kernel_sources_sha256()
    if cur != s.group(1):
        return None, "kernel changed since the ncu capture"
    return float(m.group(1)), None


# ---------------------------------------------------------------- the step

def workload_config(w, world):
    """The "config" of the JSON line, the same for both arms."""
    q_gb = w.B * w.S * w.H * w.D * 2 / 1e9
    return {"workload": w.name, "description": w.description, "B": w.B, "H": w.H, "D": w.D, "S": w.S,
            "ring_size": w.P, "chunk": w.chunk, "causal_block_size": w.causal_block_size,
            "segments": w.segments, "bias": w.bias, "parallelism": f"replicas x{world}",
            "l2": "no flush: every input tensor (%.2f GB) is larger than the 126 MB L2" % q_gb}


def run_ours(args):
    import numpy as np
    import torch

    import long_context_exact_ordered_b200 as ra
    import workloads as W

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    w = W.WORKLOADS[args.workload]
    inp = W.make_inputs(w, dev, with_grad_output=True, seed=w.seed + rank)
    q, k, v, do, bias, seg = inp["q"], inp["k"], inp["v"], inp["do"], inp["bias"], inp["seg"]
    kw = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=w.causal_block_size, ring_size=w.P)
    n_vis = ra.count_visible_pairs(w.B, w.S, w.H, w.causal_block_size, None if seg is None else seg.cpu(),
                                   None if bias is None else bias.cpu())
    fl_f, fl_b = 4.0 * w.D * n_vis, 10.0 * w.D * n_vis

    # preallocated outputs and workspaces: nothing is allocated inside the timed region
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
    grads = tuple(torch.empty_like(q) for _ in range(3))
    p0 = ra.api._params(w.S, w.chunk, w.chunk, w.causal_block_size, w.P, None)
    ws_f = ra.api._workspace(ra.workspace_size(0, q, p0, bias is not None, seg is not None), dev)
    ws_b = ra.api._workspace(ra.workspace_size(1, q, p0, bias is not None, seg is not None), dev)
    launches_per_step = 1 + 3 + (2 if (bias is not None or seg is not None) else 0)

    ev_f = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    ev_b = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    step_mode = args.mode == "step"
    fwd_only = args.mode in ("fwd", "step")
    if fwd_only:
        fl_b = 0.0
        launches_per_step = 1 + (1 if (bias is not None or seg is not None) else 0)
    if step_mode:
        # The forward as the pages' ring runs it, one ra_step per (rank, step):
        # virtual rank r keeps query block r and meets key/value block
        # (r - t) mod P at step t, merging into its own fp32 running state;
        # then ra_finalize per rank.  Every state lives in HBM, as it would on
        # a real ring rank.
        P, blk = w.P, w.S // w.P
        states = [ra.init_state(w.B, blk, w.H, w.D, dev) for _ in range(P)]
        blocks = [slice(r * blk, (r + 1) * blk) for r in range(P)]
        bias_b = [None if bias is None else bias[:, sl].contiguous() for sl in blocks]
        seg_b = [None if seg is None else seg[:, sl].contiguous() for sl in blocks]
        launches_per_step = P * P + P

    def ring_of_steps():
        for r in range(P):
            acc, m, l = states[r]
            acc.zero_()
            m.fill_(float("-inf"))
            l.zero_()
            for t in range(P):
                src = (r - t) % P
                ra.ring_step(q[:, blocks[r]], k[:, blocks[src]], v[:, blocks[src]], r * blk, src * blk, acc, m, l,
                             bias_blk=bias_b[src], seg_q=seg_b[r], seg_k=seg_b[src],
                             causal_block_size=w.causal_block_size)
            ra.finalize(acc, m, l, q.dtype, out=o[:, blocks[r]], lse=lse[:, :, blocks[r]])

    def step(prof=False):
        if step_mode:
            if prof:
                ev_f[0].record()
            ring_of_steps()
            if prof:
                ev_f[1].record()
            return
        ra.ringattention(q, k, v, bias, seg, out=o, lse=lse, workspace=ws_f, prof_events=ev_f if prof else None, **kw)
        if not fwd_only:
            ra.ringattention_backward(q, k, v, o, lse, do, bias, seg, workspace=ws_b, out=grads,
                                      prof_events=ev_b if prof else None, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ra.device_status() != 0:
        raise RuntimeError("device status word reports an error after warm-up")

    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if not str(props.uuid).startswith("GPU-") else str(props.uuid))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kern_f, kern_b = [], []
    e0.record()
    for _ in range(args.steps):
        step(prof=True)
        # per-launch kernel times: the events of this step are read after the loop
        kern_f.append((ev_f[0], ev_f[1]))
        kern_b.append((ev_b[0], ev_b[1]))
        ev_f = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        ev_b = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    ms_local = e0.elapsed_time(e1)
    status = ra.device_status()
    if status != 0:
        raise RuntimeError(f"device status word reports error {status}")
    ms = max_over_ranks(ms_local, world, dev)
    t_f = statistics.mean(a.elapsed_time(b) for a, b in kern_f)
    t_b = None if fwd_only else statistics.mean(a.elapsed_time(b) for a, b in kern_b)
    value = aggregate((fl_f + fl_b) * args.steps, ms / 1e3, world) / 1e12

    # ------------------------------------------------------------ end to end through the public API
    e2e = None
    if not args.no_e2e and not fwd_only:
        e2e = run_e2e(args, w, inp, kw, dev, n_vis, world)

    peaks, peak_src = load_peaks()
    traffic, traffic_note = traffic_per_launch()
    # the forward's co-ceiling: one MUFU ex2 per visible pair, measured live
    mr = mufu_rate(dev)
    mufu = None
    if mr is not None:
        rate, sms = mr
        mhz = (clocks or {}).get("sm_mhz") or 0
        mufu = {"ex2_per_clk_per_sm": round(rate, 2), "microbenchmark": "ra_debug_ex2_rate (libringattn_count.so)",
                "fwd_cap_tflops_at_sm_mhz": round(rate * sms * mhz * 1e6 * 4 * w.D / 1e12, 1) if mhz else None}
    fwd_tf = fl_f / (t_f / 1e3) / 1e12
    achieved = fwd_tf if fwd_only else fl_b / (t_b / 1e3) / 1e12
    if fwd_only:
        traffic, traffic_note = None, "forward kernel: see profiles/ for its ncu summary"
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    kname = "ra_fwd_sm100_kernel" if fwd_only else "ra_bwd_sm100_kernel"
    roofline = {"bound": "tensor", "kernel": kname, "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a multi-second loop)",
                "frac_of_burst_peak": round(achieved / burst, 4), "traffic": traffic,
                "dram_gbs": (round(traffic / (t_b / 1e3) / 1e9, 1) if traffic is not None and t_b else None),
                "traffic_note": traffic_note or "dram bytes per launch from the committed ncu capture",
                "algorithmic_flop_per_launch": fl_f if fwd_only else fl_b}
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
        "config": workload_config(w, world),
        "mode": ("forward as P*P ring steps (ra_step) + finalize" if step_mode else
                 "forward only" if fwd_only else "forward + backward"),
        "fwd_tflops": round(fwd_tf, 2), "bwd_tflops": None if fwd_only else round(achieved, 2),
        "frac_of_burst_peak_fwd_bwd": round(value / world / burst, 4),
        "clocks": clocks, "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "roofline": roofline,
        "mufu": mufu,
        "visible_pairs": n_vis,
    }
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        out["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_ffn(args):
    """--mode ffn: the blockwise feed-forward network (ra_feedforward, SwiGLU) over
    the workload's tokens: T = B*S tokens of d_model = H*D, d_ff = 11008 (the
    LLaMA-7B ratio for d_model 4096), chunk of 8192 tokens.  Algorithmic
    work 6*T*d_model*d_ff flop (three products)."""
    import torch

    import long_context_exact_ordered_b200 as ra
    import workloads as W

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    w = W.WORKLOADS[args.workload]
    T, dm, dff, chunk = w.B * w.S, w.H * w.D, args.ffn_dff, args.ffn_chunk
    g = torch.Generator(device=dev).manual_seed(w.seed + rank)
    x = torch.randn((T, dm), generator=g, device=dev).to(torch.bfloat16)
    w1 = (torch.randn((dff, dm), generator=g, device=dev) * dm ** -0.5).to(torch.bfloat16)
    w3 = (torch.randn((dff, dm), generator=g, device=dev) * dm ** -0.5).to(torch.bfloat16)
    w2 = (torch.randn((dm, dff), generator=g, device=dev) * dff ** -0.5).to(torch.bfloat16)
    y = torch.empty_like(x)
    ws = torch.empty(ra.load().ra_feedforward_workspace_size(chunk, dff), dtype=torch.uint8, device=dev)
    step = lambda: ra.blockwise_feedforward(x, w1, w3, w2, chunk_size=chunk, out=y, workspace=ws)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if not str(props.uuid).startswith("GPU-") else str(props.uuid))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    fl = 6.0 * T * dm * dff
    value = aggregate(fl * args.steps, ms / 1e3, world) / 1e12
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    n_chunks = (T + chunk - 1) // chunk
    out = {
        "metric": "blockwise feed-forward TFLOP/s", "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
        "config": {"workload": f"ffn_{w.name}", "tokens": T, "d_model": dm, "d_ff": dff, "chunk": chunk,
                   "parallelism": f"replicas x{world}",
                   "l2": "no flush: the weights (%.2f GB) and activations exceed the 126 MB L2" % (3 * dm * dff * 2 / 1e9)},
        "mode": "blockwise feed-forward (SwiGLU)", "clocks": clocks, "e2e": None,
        "gpu_launches": 2 * n_chunks * args.steps,
        "roofline": {"bound": "tensor", "kernel": "ra_ffn_gemm_kernel", "achieved": round(value / world, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(value / world / peak, 4),
                     "frac_of_burst_peak": round(value / world / burst, 4),
                     "peak_source": f"{peak_src} bf16_tflops_sustained", "traffic": None},
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_ring(args):
    """--ring: the forward with the sequence sharded over the N ranks, key/value
    blocks exchanged round the ring over NCCL (long_context_exact_ordered_b200.ring,
    zig-zag layout), ra_step on each rank's tensor cores.  Total work is fixed
    ("scaling": "strong"); the value is the whole sequence's algorithmic
    forward FLOP over the slowest rank's device time."""
    import torch

    import long_context_exact_ordered_b200 as ra
    from long_context_exact_ordered_b200 import ring
    import workloads as W

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    w = W.WORKLOADS[args.workload]
    full = W.make_inputs(w, dev, with_grad_output=False)
    n_vis = ra.count_visible_pairs(w.B, w.S, w.H, w.causal_block_size,
                                   None if full["seg"] is None else full["seg"].cpu(),
                                   None if full["bias"] is None else full["bias"].cpu())
    mine = {n: (None if full[n] is None else ring.shard(full[n], rank, world, "zigzag"))
            for n in ("q", "k", "v", "bias", "seg")}
    del full
    torch.cuda.empty_cache()
    comm = torch.cuda.Stream(dev)

    def step():
        return ring.ring_attention_forward(mine["q"], mine["k"], mine["v"], mine["bias"], mine["seg"],
                                           causal_block_size=w.causal_block_size, layout="zigzag",
                                           comm_stream=comm)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ra.device_status() != 0:
        raise RuntimeError("device status word reports an error after warm-up")
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if not str(props.uuid).startswith("GPU-") else str(props.uuid))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    fl = 4.0 * w.D * n_vis
    value = fl * args.steps / (ms / 1e3) / 1e12
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    per_gpu = value / world
    calls = 4 * world + 2                  # ra_step calls (two query x two key chunks per ring step) + finalize
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "D": w.D, "S": w.S, "causal_block_size": w.causal_block_size,
                   "segments": w.segments, "parallelism": f"ring x{world} (sequence sharded, zig-zag, NCCL P2P)",
                   "l2": "no flush: every rank's K / V shard is larger than the 126 MB L2" if w.S // world * w.H * w.D * 2 > 126e6
                   else "no flush (small shards)"},
        "mode": "ring forward across ranks", "clocks": clocks, "e2e": None,
        "gpu_launches": calls * args.steps,
        "roofline": {"bound": "tensor", "kernel": "ra_fwd_sm100_kernel (ring-step mode)", "achieved": round(per_gpu, 2),
                     "peak": burst, "unit": "TFLOP/s", "frac": round(per_gpu / burst, 4),
                     "peak_source": f"{peak_src} bf16_tflops (burst)", "traffic": None},
        "visible_pairs": n_vis,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_e2e(args, w, inp, kw, dev, n_vis, world):
    """Same metric through the public host-buffer API (HostStep -> ra_train_step_host):
    every step copies q, k, v, dO from pinned host memory and o, lse, dq, dk, dv
    back, overlapped with the kernels by head groups."""
    import torch

    import long_context_exact_ordered_b200 as ra

    names = ("q", "k", "v", "do")
    host = {n: inp[n].cpu().pin_memory() for n in names}
    outs_h = [torch.empty(inp["q"].shape, dtype=inp["q"].dtype, pin_memory=True) for _ in range(4)]
    lse_h = torch.empty((w.B, w.H, w.S), dtype=torch.float32, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h) + lse_h.numel() * 4
    step = ra.HostStep(w.B, w.S, w.H, w.D, dtype=inp["q"].dtype, device=dev, has_bias=inp["bias"] is not None,
                       has_segments=inp["seg"] is not None, **kw)

    def one():
        step(host["q"], host["k"], host["v"], host["do"], outs_h[0], lse_h, outs_h[1], outs_h[2], outs_h[3],
             attention_bias=inp["bias"], segment_ids=inp["seg"])

    one()
    torch.cuda.synchronize()
    n = max(1, args.steps)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        one()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    val = aggregate(14.0 * w.D * n_vis * n, ms / 1e3, world) / 1e12
    hpg = step.hpg
    del step
    return {"value": round(val, 2), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "ms_per_step": round(ms / n, 3),
            "api": "HostStep / ra_train_step_host: host-buffer fwd+bwd, copies overlapped by head groups",
            "heads_per_group": hpg}


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)

_ORACLE_INPUTS = {}


def oracle_sample(w, rows_per_head, heads, seed):
    """Oracle forward + backward for a bounded sample of query rows: the float64
    forward of those rows and their full backward contributions (dQ rows and
    their share of dK / dV).  Returns (seconds, visible pairs processed)."""
    import numpy as np
    import torch

    import oracle
    from oracle.attention import _head_backward
    import workloads as W

    rng = np.random.default_rng(seed)
    if w.name not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[w.name] = W.make_inputs(w, "cpu", with_grad_output=True)
    inp = _ORACLE_INPUTS[w.name]
    pairs = 0
    # the inputs of a head, upcast to float64 once and kept (like the GPU's
    # inputs resident in HBM); the oracle's own work is all that is timed
    for h in heads:
        if (w.name, h) not in _ORACLE_INPUTS:
            _ORACLE_INPUTS[(w.name, h)] = tuple(inp[n][0, :, h].float().double().numpy() for n in ("q", "k", "v", "do"))
    t0 = time.perf_counter()
    for h in heads:
        qh, kh, vh, doh = _ORACLE_INPUTS[(w.name, h)]
        rows = np.sort(rng.choice(w.S, size=rows_per_head, replace=False))
        seg_b = None if inp["seg"] is None else inp["seg"][0].numpy()
        sub = np.stack([np.zeros_like(rows), np.zeros_like(rows), rows], axis=1)
        o_r, lse_r = oracle.attention_rows(None, kh[None, :, None], vh[None, :, None], sub, None,
                                           None if seg_b is None else seg_b[None], w.causal_block_size,
                                           q_rows=qh[rows])
        _head_backward(qh[rows], kh, vh, doh[rows], o_r, lse_r, rows, w.causal_block_size, seg_b, None)
        pairs += int(oracle.visible_count_rows(rows, w.S, w.causal_block_size, seg_b).sum())
    return time.perf_counter() - t0, pairs


def blas_threads():
    try:
        import threadpoolctl

        return max(i["num_threads"] for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas")
    except Exception:
        return len(os.sched_getaffinity(0))


def calibrate_rows(w, budget_s):
    """Query rows of head 0 that the oracle processes in about ``budget_s`` seconds
    (two-point fit: a fixed cost per call plus a cost per row)."""
    oracle_sample(w, 8, [0], seed=0)            # loads and upcasts the head's inputs once
    t8, _ = oracle_sample(w, 8, [0], seed=1)
    t64, _ = oracle_sample(w, 64, [0], seed=1)
    per_row = max((t64 - t8) / 56, 1e-6)
    return int(max(8, min(8192, (budget_s - t8) / per_row)))


def cpu_baseline(w, budget_s=20.0):
    """The oracle as it stands on this host's cores, on a bounded sample of the workload."""
    rows = calibrate_rows(w, budget_s)
    secs, pairs = oracle_sample(w, rows, [0], seed=2)
    val = 14.0 * w.D * pairs / secs / 1e12
    return {"value": val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} random query rows of head 0 of {w.name}: float64 forward rows + their full backward "
                      f"({pairs} visible pairs, {secs:.1f} s)"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import workloads as W

    w = W.WORKLOADS[args.workload]
    # rows per step: about --ref-step-seconds of oracle work each (unless --ref-rows is given)
    rows = args.ref_rows if args.ref_rows else calibrate_rows(w, args.ref_step_seconds)
    for i in range(args.warmup):
        oracle_sample(w, rows, [0], seed=100 + i)
    secs, pairs = 0.0, 0
    for i in range(args.steps):
        s, p = oracle_sample(w, rows, [0], seed=200 + i)
        secs += s
        pairs += p
    val = 14.0 * w.D * pairs / secs / 1e12
    cores = blas_threads()
    sample = f"{rows} random query rows of head 0 per step: float64 forward rows + their full backward"
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) bf16)",
           "config": workload_config(w, world),
           "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="causal128k")
    ap.add_argument("--ffn-dff", type=int, default=11008, help="--mode ffn: hidden width d_ff")
    ap.add_argument("--ffn-chunk", type=int, default=8192, help="--mode ffn: tokens per chunk")
    ap.add_argument("--mode", choices=["fwdbwd", "fwd", "step", "ffn"], default="fwdbwd",
                    help="fwdbwd: one step = forward + backward (default); fwd: forward only; step: the forward "
                         "as P*P per-step calls (ra_step, tensor cores) plus ra_finalize per rank; ffn: the "
                         "blockwise feed-forward network over the workload's tokens")
    ap.add_argument("--ring", action="store_true",
                    help="forward with the sequence sharded over the N ranks (ring of NCCL exchanges) instead of "
                         "N independent replicas")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="query rows per reference-arm step (0: calibrated to --ref-step-seconds)")
    ap.add_argument("--ref-step-seconds", type=float, default=4.0,
                    help="oracle seconds per reference-arm step when calibrating the sample")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.ring:
        run_ring(args)
    elif args.mode == "ffn":
        run_ffn(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
