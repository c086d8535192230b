"""Benchmark of the one-GPU Ulysses attention layer (repack -> attention -> inverse repack).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config long104k] [--impl ours|reference]

One step = one pass of the whole layer over the workload's synthetic input:
ulysses_repack_fwd (all planes) -> ulysses_attn_fwd -> ulysses_repack_bwd
(output plane), each a C-ABI call on one stream with CUDA events between
them.  Rank 0 prints one JSON line.  N > 1 runs N independent replicas (the
layer has no exchange between GPUs in this build), launched with torchrun;
the job then processes N layers per step, so ``value`` (and ``e2e.value``)
is the slowest rank's step time divided by N, the whole job's time per
layer, with the per-replica time in ``per_replica_us``.

The default workload is the largest one that fits one GPU, the long clip
(P=8, N=104,448, H=56).  The line also carries the other layer workloads
(Video-DiT, the QKVG clip and the varlen long clip), each timed over a few
steps after the main timed region.

``--impl reference`` times the CPU oracle instead, on a bounded sample of
the same workload per step, extrapolated to the full layer (the same sample
definition as the ``cpu_baseline`` of the main arm).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# name: (P, N, H, planes, seed, cu_seqlens)
WORKLOADS = {
    "tiny": (2, 1024, 8, 3, 0, None),
    "dit19k": (4, 19_394, 56, 3, 1, None),
    "clip38k": (4, 38_912, 56, 4, 2, None),
    "long104k": (8, 104_448, 56, 3, 3, None),
    "long104k-varlen": (8, 104_448, 56, 3, 3, [0, 52_224, 83_456, 104_448]),
    "prof8k": (4, 8192, 56, 3, 1, None),   # small case for profiler captures (352 MB input > L2)
    "stress250k": (4, 250_000, 56, 4, 4, None),   # repack fwd + bwd only, plus an N sweep
    "dit19k-causal": (4, 19_394, 56, 3, 1, None),
    "dit19k-fp8": (4, 19_394, 56, 3, 1, None),
    "prof8k-fp8": (4, 8192, 56, 3, 1, None),   # small FP8 case for profiler captures
}
CAUSAL = {"dit19k-causal"}
FP8 = {"dit19k-fp8", "prof8k-fp8"}
SWEEP_N = (4096, 8192, 16384, 32768, 65536, 131072, 250_000)
WORKLOAD_TEXT = {
    "tiny": "Tiny Ulysses layer P=2 N=1024 H=8 D=128 packed QKV bf16",
    "dit19k": "Video-DiT geometry P=4 N=19394 H=56 D=128 packed QKV bf16 [N,3,H,D]",
    "clip38k": "Longer clip P=4 N=38912 H=56 D=128 packed QKVG bf16 [N,4,H,D]",
    "long104k": "Long clip P=8 N=104448 H=56 D=128 packed QKV bf16",
    "long104k-varlen": "Long clip varlen P=8 N=104448 H=56 D=128, 3 sequences 52224/31232/20992",
    "prof8k": "Profiling case P=4 N=8192 H=56 D=128 packed QKV bf16",
    "stress250k": "Repack stress P=4 N=250000 H=56 D=128 packed QKVG bf16, one 896,000,000-byte plane per rank "
                  "per launch; repack fwd+bwd; N sweep 4096..250000",
    "dit19k-causal": "Video-DiT geometry with causal attention P=4 N=19394 H=56 D=128 packed QKV bf16",
    "prof8k-fp8": "Profiling case, FP8 variant, P=4 N=8192 H=56 D=128 packed QKV bf16 in and out",
    "dit19k-fp8": "Video-DiT geometry, FP8 variant: Q/K/V cast to E4M3 in the repack, E4M3 attention, "
                  "P=4 N=19394 H=56 D=128 packed QKV bf16 in and out",
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def pct(xs, q):
    """q-th percentile (nearest rank) of a list of per-step times."""
    ys = sorted(xs)
    return ys[min(len(ys) - 1, max(0, math.ceil(q / 100.0 * len(ys)) - 1))]


def tensor_peak(pk):
    """Dense bf16 denominator for the attention kernel: the measured cuBLAS
    burst figure.  It is the larger of the two measured GEMM figures, so the
    fraction against it is the conservative one.  Long launches run under
    the 1 kW power cap, where the clock falls below the burst GEMM's; the
    fraction of the sustained (power-capped) GEMM figure is reported beside
    it, never instead of it."""
    return pk["bf16_tflops"], "bf16 burst"


def sustained_peak(pk):
    return pk.get("bf16_tflops_sustained", pk["bf16_tflops"])


def attn_flops(N, H, cu, causal=False):
    segs = [(0, N)] if cu is None else list(zip(cu, cu[1:]))
    if causal:
        return float(sum(4 * H * 128 * (b - a) * (b - a + 1) // 2 for a, b in segs))
    return float(sum(4 * (b - a) ** 2 * H * 128 for a, b in segs))


def source_hash(name):
    p = os.path.join(ROOT, "ulysses_sequence_attention_repack_b200", "csrc", name)
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    rec = d.get(kernel, {}).get(workload)
    if not rec or rec.get("source_sha256_16") != source_hash(rec["source"]):
        return None
    return rec["dram_bytes_per_launch"]


class ClockSampler:
    """nvidia-smi sampled every 100 ms around the timed region; the clock,
    power and throttle reasons are taken from the samples that fall between
    begin() and end() (the host calls bracketing the timed GPU work)."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu_index = gpu_index
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def begin(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    @staticmethod
    def _stamp(text):
        import datetime
        try:
            return datetime.datetime.strptime(text, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [[x.strip() for x in line.split(",")] for line in out.strip().splitlines() if line.strip()]
        samples = []
        for r in rows:
            if len(r) < 8:
                continue
            try:
                samples.append((self._stamp(r[0]), float(r[1]), float(r[2]), float(r[3]), r[4:8]))
            except ValueError:
                continue
        inside = [x for x in samples if x[0] is not None and self.t0 is not None and self.t1 is not None
                  and self.t0 <= x[0] <= self.t1]
        window = "timed region"
        if not inside:            # region shorter than one sampling period: the loaded samples
            top = max((x[3] for x in samples), default=0.0)
            inside = [x for x in samples if x[3] >= 0.6 * top]
            window = "samples at >= 60% of the peak power seen"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for x in inside for n, v in zip(names, x[4]) if v.lower() == "active"})
        mx = samples[-1][2] if samples else None
        return {"sm_mhz": statistics.median(x[1] for x in inside) if inside else None, "sm_max_mhz": mx,
                "power_w": statistics.median(x[3] for x in inside) if inside else None,
                "reasons": reasons, "samples": len(inside), "window": window}


# ---------------------------------------------------------------------------- our arm

OTHER_WORKLOADS = ("dit19k", "clip38k", "long104k-varlen")


def time_layer_workload(U, inputs, name, dev, stream, steps, warmup=3):
    """Layer, attention and repack times of one more workload (the main
    step's call sequence), for the line's ``workloads`` sub-dict."""
    import torch
    P, N, H, C, seed, cu = WORKLOADS[name]
    causal = name in CAUSAL
    plan = U.ulysses_plan(N, H, 128, P, C, 0, 0, 0, cu, causal=causal)
    Np, Hl = plan.padded_tokens, H // P
    S = inputs.qkv_seq(N, H, P, C, seed, dev)
    T = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=dev)
    scale = 1.0 / math.sqrt(128)
    for _ in range(warmup):
        U.ulysses_repack_fwd(plan, S, T, stream)
        U.ulysses_attn_fwd(plan, T, OT, scale, stream)
        U.ulysses_repack_bwd(plan, OT, OS, 1, stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for e in evs:
        e[0].record(stream)
        U.ulysses_repack_fwd(plan, S, T, stream)
        e[1].record(stream)
        U.ulysses_attn_fwd(plan, T, OT, scale, stream)
        e[2].record(stream)
        U.ulysses_repack_bwd(plan, OT, OS, 1, stream)
        e[3].record(stream)
    torch.cuda.synchronize()
    if U.ulysses_last_device_error(plan) != 0:
        raise RuntimeError(f"a kernel reported a device error in the {name} workload")
    layer = statistics.mean(e[0].elapsed_time(e[3]) for e in evs)
    at = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    rf = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    rb = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    tflops = attn_flops(N, H, cu, causal) / (at * 1e-3) / 1e12
    return {"workload": WORKLOAD_TEXT[name], "steps": steps, "layer_us": round(layer * 1000, 2),
            "attn_us": round(at * 1000, 2), "attn_tflops": round(tflops, 1),
            "repack_fwd_gbs": round(2 * C * Np * H * 128 * 2 / (rf * 1e-3) / 1e9, 1),
            "repack_bwd_gbs": round(2 * Np * H * 128 * 2 / (rb * 1e-3) / 1e9, 1)}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    P, N, H, C, seed, cu = WORKLOADS[args.config]
    causal = args.config in CAUSAL
    Hl = H // P
    plan = U.ulysses_plan(N, H, 128, P, C, 0, 0, 0, cu, causal=causal, pair_cta=args.pair_attention)
    Np = plan.padded_tokens
    S = inputs.qkv_seq(N, H, P, C, seed, dev)
    T = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    scale = 1.0 / math.sqrt(128)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        U.ulysses_repack_fwd(plan, S, T, stream)
        if evs:
            evs[1].record(stream)
        U.ulysses_attn_fwd(plan, T, OT, scale, stream)
        if evs:
            evs[2].record(stream)
        U.ulysses_repack_bwd(plan, OT, OS, 1, stream)
        if evs:
            evs[3].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    sampler.begin()
    start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    stop.record(stream)
    torch.cuda.synchronize()
    sampler.end()
    barrier()
    clocks = sampler.stop()
    total_ms = start.elapsed_time(stop)
    t_rf = [e[0].elapsed_time(e[1]) for e in evs]
    t_at = [e[1].elapsed_time(e[2]) for e in evs]
    t_rb = [e[2].elapsed_time(e[3]) for e in evs]
    t_step = [e[0].elapsed_time(e[3]) for e in evs]
    if U.ulysses_last_device_error(plan) != 0:
        raise RuntimeError("a kernel reported a device error during the timed region")

    # fused variant (attention reads the sequence-sharded input directly), timed right
    # after the unfused steps and over as many steps, so both see the same power state
    for _ in range(3):
        U.ulysses_layer_fwd(plan, S, OS, None, fused=1, stream=stream)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nf = args.steps
    f0.record(stream)
    for _ in range(nf):
        U.ulysses_layer_fwd(plan, S, OS, None, fused=1, stream=stream)
    f1.record(stream)
    torch.cuda.synchronize()
    fused_ms = f0.elapsed_time(f1) / nf

    # the multi-GPU push path with its P ranks emulated on this GPU: each rank
    # pushes its shard (rows of S) into every head slab (slabs of T), then each
    # rank's attention stores its rows into the owners' output shards (rows of OS)
    Nl = plan.rows_per_rank
    shards = [S[q * Nl:(q + 1) * Nl] for q in range(P)]
    slabs = [T[r] for r in range(P)]
    outs = [OS[q * Nl:(q + 1) * Nl] for q in range(P)]

    def push_layer(evs=None):
        if evs:
            evs[0].record(stream)
        for q in range(P):
            U.ulysses_repack_fwd_push(plan, q, shards[q], slabs, stream=stream)
        if evs:
            evs[1].record(stream)
        for r in range(P):
            U.ulysses_attn_fwd_push(plan, r, slabs[r], outs, scale, stream)
        if evs:
            evs[2].record(stream)

    for _ in range(3):
        push_layer()
    pevs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for k in range(args.steps):
        push_layer(pevs[k])
    torch.cuda.synchronize()
    push_ms = statistics.mean(e[0].elapsed_time(e[2]) for e in pevs)
    push_rf_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in pevs)
    if U.ulysses_last_device_error(plan) != 0:
        raise RuntimeError("a kernel reported a device error in the push path")

    # step 1 with the QKV prologue fused in (RMSNorm + partial RoPE on Q and K,
    # rotary_dim 96 as in the pages), timed on the same input
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 500)
    wq = torch.randn(128, generator=g, device=dev).to(torch.bfloat16)
    wk = torch.randn(128, generator=g, device=dev).to(torch.bfloat16)
    ang = torch.rand((Np, 48), generator=g, device=dev) * 6.2832
    cos_t = torch.cat([torch.cos(ang), torch.cos(ang)], 1).to(torch.bfloat16).contiguous()
    sin_t = torch.cat([torch.sin(ang), torch.sin(ang)], 1).to(torch.bfloat16).contiguous()
    for _ in range(3):
        U.ulysses_prologue_repack_fwd(plan, S, T, wq, wk, cos_t, sin_t, 96, 1e-5, stream)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    npro = max(3, args.steps)
    p0.record(stream)
    for _ in range(npro):
        U.ulysses_prologue_repack_fwd(plan, S, T, wq, wk, cos_t, sin_t, 96, 1e-5, stream)
    p1.record(stream)
    torch.cuda.synchronize()
    prologue_ms = p0.elapsed_time(p1) / npro

    # training direction: forward with lse, then the attention backward
    # (algorithmic FLOPs 2.5x the forward's: dV, dP, dQ, dK plus S recomputed)
    lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=dev)
    dO = torch.randn(OT.shape, generator=g, device=dev).to(torch.bfloat16)
    dT = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
    bws = torch.empty(plan.attn_bwd_workspace_bytes, dtype=torch.uint8, device=dev)
    U.ulysses_attn_fwd_lse(plan, T, OT, lse, scale, stream)
    for _ in range(2):
        U.ulysses_attn_bwd(plan, T, OT, dO, lse, dT, bws, scale, stream=stream)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nbw = max(3, args.steps // 3)
    b0.record(stream)
    for _ in range(nbw):
        U.ulysses_attn_bwd(plan, T, OT, dO, lse, dT, bws, scale, stream=stream)
    b1.record(stream)
    torch.cuda.synchronize()
    bwd_ms = b0.elapsed_time(b1) / nbw
    if U.ulysses_last_device_error(plan) != 0:
        raise RuntimeError("a kernel reported a device error in the backward")
    # the deterministic two-pass backward (ULYSSES_PLAN_DETERMINISTIC) on the same inputs
    dplan = U.ulysses_plan(N, H, 128, P, C, 0, 0, 0, cu, causal=causal, deterministic=True)
    del bws
    bws = torch.empty(dplan.attn_bwd_workspace_bytes, dtype=torch.uint8, device=dev)
    for _ in range(2):
        U.ulysses_attn_bwd(dplan, T, OT, dO, lse, dT, bws, scale, stream=stream)
    b0.record(stream)
    for _ in range(nbw):
        U.ulysses_attn_bwd(dplan, T, OT, dO, lse, dT, bws, scale, stream=stream)
    b1.record(stream)
    torch.cuda.synchronize()
    bwd_det_ms = b0.elapsed_time(b1) / nbw
    if U.ulysses_last_device_error(dplan) != 0:
        raise RuntimeError("a kernel reported a device error in the deterministic backward")
    del bws

    # end to end through the C ABI from pinned host buffers
    host_in = S.cpu().pin_memory()
    host_out = torch.empty(OS.shape, dtype=OS.dtype).pin_memory()
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
    dev_in = torch.empty_like(S)
    for _ in range(2):
        U.ulysses_layer_fwd_host(plan, host_in, host_out, dev_in, OS, ws, fused=0, stream=stream)
    torch.cuda.synchronize()
    ne = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    for _ in range(ne):
        U.ulysses_layer_fwd_host(plan, host_in, host_out, dev_in, OS, ws, fused=0, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / ne
    h2d = host_in.numel() * host_in.element_size()
    d2h = host_out.numel() * host_out.element_size()

    # the other layer workloads, a few steps each (outside the timed region)
    others = {}
    if not args.no_other_workloads:
        del host_in, host_out, dev_in, ws, lse, dO, dT
        for name in OTHER_WORKLOADS:
            if name != args.config:
                others[name] = time_layer_workload(U, inputs, name, dev, stream, steps=max(3, min(args.steps, 10)))
                torch.cuda.empty_cache()

    vals = torch.tensor([total_ms, e2e_ms, fused_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    total_ms, e2e_ms, fused_ms = vals.tolist()
    if rank != 0:
        return None

    pk, pk_kind = peaks()
    flops = attn_flops(N, H, cu, causal)
    at_ms = statistics.mean(t_at)
    rf_ms, rb_ms = statistics.mean(t_rf), statistics.mean(t_rb)
    rf_bytes = 2 * C * Np * H * 128 * 2
    rb_bytes = 2 * Np * H * 128 * 2
    attn_tflops = flops / (at_ms * 1e-3) / 1e12
    rf_gbs = rf_bytes / (rf_ms * 1e-3) / 1e9
    rb_gbs = rb_bytes / (rb_ms * 1e-3) / 1e9
    ms_per_step = total_ms / args.steps
    launches_per_step = math.ceil(C / plan.plane_chunk) + 1 + 1
    traffic = recorded_traffic("attn_fwd_pair_kernel" if args.pair_attention else "attn_fwd_kernel", args.config)
    tpk, tpk_kind = tensor_peak(pk)
    spk = sustained_peak(pk)
    for w in others.values():
        w["attn_frac_of_burst"] = round(w["attn_tflops"] / tpk, 3)
        w["repack_fwd_frac"] = round(w["repack_fwd_gbs"] / pk["hbm_gbs"], 3)
    line = {
        "metric": "Ulysses layer µs; attn TFLOP/s and repack GB/s vs B200 peak",
        # N replicas process N layers per step: the job's time per layer is the
        # slowest rank's step time over N (per-replica time in per_replica_us)
        "value": round(ms_per_step * 1000.0 / world, 2),
        "unit": "us per layer",
        "n_gpus": world,
        "per_replica_us": round(ms_per_step * 1000.0, 2),
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic N(0,1) bf16, seeded",
        "config": {"workload": WORKLOAD_TEXT[args.config], "name": args.config, "P": P, "N": N, "Np": Np,
                   "H": H, "D": 128, "planes": C, "seed": seed, "cu_seqlens": cu, "causal": causal,
                   "step": "repack_fwd + attn_fwd + repack_bwd(output), one C-ABI call each",
                   "attention_kernel": "CTA pairs" if args.pair_attention else "one CTA per SM",
                   "replicas": world, "l2": f"inputs larger than L2 ({S.numel() * 2 / 1e6:.0f} MB per step)"},
        "attn_us": round(at_ms * 1000, 2),
        "attn_tflops": round(attn_tflops, 1),
        "per_step_us": {"layer_p50": round(pct(t_step, 50) * 1000, 2), "layer_p95": round(pct(t_step, 95) * 1000, 2),
                        "attn_p50": round(pct(t_at, 50) * 1000, 2), "attn_p95": round(pct(t_at, 95) * 1000, 2)},
        "repack_fwd_us": round(rf_ms * 1000, 2),
        "repack_fwd_gbs": round(rf_gbs, 1),
        "repack_bwd_us": round(rb_ms * 1000, 2),
        "repack_bwd_gbs": round(rb_gbs, 1),
        "repack_fwd_frac": {"measured": round(rf_gbs / pk["hbm_gbs"], 3),
                            "spec_8TBs": round(rf_gbs / SPEC_PEAKS["hbm_gbs"], 3)},
        "attn_frac": {"measured_burst": round(attn_tflops / pk["bf16_tflops"], 3),
                      "measured_sustained": round(attn_tflops / spk, 3),
                      "spec_2250": round(attn_tflops / SPEC_PEAKS["bf16_tflops"], 3)},
        "fused_layer_us": round(fused_ms * 1000, 2),
        "push_layer_us": round(push_ms * 1000, 2),
        "push_repack_fwd_gbs": round(rf_bytes / (push_rf_ms * 1e-3) / 1e9, 1),
        "attn_bwd_us": round(bwd_ms * 1000, 2),
        "attn_bwd_tflops": round(2.5 * flops / (bwd_ms * 1e-3) / 1e12, 1),
        "attn_bwd_deterministic_us": round(bwd_det_ms * 1000, 2),
        "prologue_repack_fwd_us": round(prologue_ms * 1000, 2),
        "prologue_repack_fwd_gbs": round(rf_bytes / (prologue_ms * 1e-3) / 1e9, 1),
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_pair_kernel" if args.pair_attention else "attn_fwd_kernel",
                     "achieved": round(attn_tflops, 1),
                     "peak": tpk, "peak_kind": f"{pk_kind} {tpk_kind}", "unit": "TFLOP/s",
                     "frac": round(attn_tflops / tpk, 3),
                     "frac_of_sustained": round(attn_tflops / spk, 3), "traffic": traffic,
                     "algorithmic_flops_per_launch": flops},
        "e2e": {"value": round(e2e_ms * 1000 / world, 2), "unit": "us per layer", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "path": "ulysses_layer_fwd_host (pinned host in/out)",
                "per_replica_us": round(e2e_ms * 1000, 2)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "workloads": others,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.config, S)
    return line


def run_fp8(args, rank, world, local_rank):
    """The FP8 layer: repack with the E4M3 cast -> E4M3 attention -> inverse repack (bf16 output)."""
    import torch
    import torch.distributed as dist
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    P, N, H, C, seed, cu = WORKLOADS[args.config]
    Hl = H // P
    plan = U.ulysses_plan(N, H, 128, P, C, 0, 0, 0, cu)
    Np = plan.padded_tokens
    S = inputs.qkv_seq(N, H, P, C, seed, dev)
    T8 = torch.empty((P, C, Np, Hl, 128), dtype=torch.uint8, device=dev)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    scale = 1.0 / math.sqrt(128)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        U.ulysses_repack_fwd_fp8(plan, S, T8, stream)
        if evs:
            evs[1].record(stream)
        U.ulysses_attn_fwd_fp8(plan, T8, OT, scale, stream)
        if evs:
            evs[2].record(stream)
        U.ulysses_repack_bwd(plan, OT, OS, 1, stream)
        if evs:
            evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.begin()
    start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    stop.record(stream)
    torch.cuda.synchronize()
    sampler.end()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    if U.ulysses_last_device_error(plan) != 0:
        raise RuntimeError("a kernel reported a device error during the timed region")
    total_ms = start.elapsed_time(stop)

    # end to end through the C ABI from pinned host buffers, streamed by head groups
    host_in = S.cpu().pin_memory()
    host_out = torch.empty(OS.shape, dtype=OS.dtype).pin_memory()
    dev_in = torch.empty_like(S)
    ws = torch.empty(plan.workspace_bytes_fp8, dtype=torch.uint8, device=dev)
    ne = max(3, min(args.steps, 10))
    for _ in range(2):
        U.ulysses_layer_fwd_fp8_host(plan, host_in, host_out, dev_in, OS, ws, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(ne):
        U.ulysses_layer_fwd_fp8_host(plan, host_in, host_out, dev_in, OS, ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / ne

    vals = torch.tensor([total_ms, e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    total_ms, e2e_ms = vals.tolist()
    if rank != 0:
        return None
    pk, pk_kind = peaks()
    # measured bf16 x the nominal fp8/bf16 ratio (4.5 / 2.25).  The burst figure:
    # this kernel draws less power and holds 1.78-1.84 GHz under back-to-back
    # launches (measured inside the kernel), the clock regime of the burst GEMM
    fp8_peak = 2.0 * pk["bf16_tflops"]
    flops = attn_flops(N, H, cu)
    at_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    rf_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    rb_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    rf_bytes = C * Np * H * 128 * 3          # read bf16, write E4M3
    rb_bytes = 2 * Np * H * 128 * 2
    attn_tflops = flops / (at_ms * 1e-3) / 1e12
    ms_per_step = total_ms / args.steps
    return {
        "metric": "Ulysses layer µs; attn TFLOP/s and repack GB/s vs B200 peak",
        "value": round(ms_per_step * 1000.0 / world, 2), "unit": "us per layer", "n_gpus": world,
        "per_replica_us": round(ms_per_step * 1000.0, 2), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 attention, bf16 in/out",
        "data": "synthetic N(0,1) bf16, seeded",
        "config": {"workload": WORKLOAD_TEXT[args.config], "name": args.config, "P": P, "N": N, "Np": Np, "H": H,
                   "D": 128, "planes": C, "seed": seed,
                   "step": "repack_fwd_fp8 + attn_fwd_fp8 + repack_bwd(output), one C-ABI call each",
                   "replicas": world, "l2": f"inputs larger than L2 ({S.numel() * 2 / 1e6:.0f} MB per step)"},
        "attn_us": round(at_ms * 1000, 2), "attn_tflops": round(attn_tflops, 1),
        "repack_fwd_fp8_us": round(rf_ms * 1000, 2),
        "repack_fwd_fp8_gbs": round(rf_bytes / (rf_ms * 1e-3) / 1e9, 1),
        "repack_bwd_us": round(rb_ms * 1000, 2), "repack_bwd_gbs": round(rb_bytes / (rb_ms * 1e-3) / 1e9, 1),
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel<fp8>", "achieved": round(attn_tflops, 1),
                     "peak": round(fp8_peak, 1), "peak_kind": f"{pk_kind} bf16 burst x 2 (E4M3 dense)",
                     "unit": "TFLOP/s", "frac": round(attn_tflops / fp8_peak, 3),
                     "frac_of_sustained": round(attn_tflops / (2.0 * pk.get("bf16_tflops_sustained",
                                                                            pk["bf16_tflops"])), 3),
                     "traffic": recorded_traffic("attn_fwd_kernel_fp8", args.config),
                     "algorithmic_flops_per_launch": flops},
        "e2e": {"value": round(e2e_ms * 1000 / world, 2), "unit": "us per layer",
                "h2d_bytes_per_step": host_in.numel() * 2, "d2h_bytes_per_step": host_out.numel() * 2,
                "path": "ulysses_layer_fwd_fp8_host (pinned host in/out)", "per_replica_us": round(e2e_ms * 1000, 2)},
        "gpu_launches": (math.ceil(C / plan.plane_chunk) + 2) * args.steps,
        "clocks": clocks,
    }


def run_transport(args, rank, world, local_rank):
    """Opt-in (--transport peer|nccl): the layer across the N GPUs of the
    launch, one rank per GPU, rank q holding rows [q*Nl, (q+1)*Nl) of the
    workload: PeerLayer (pushes over peer memory, the inverse exchange fused
    into attention) or CollectiveLayer (NCCL all-to-all around this library's
    pack/unpack kernels).  The plan's P is the number of GPUs; the total
    problem is fixed (strong scaling)."""
    import torch
    import torch.distributed as dist
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs, peer

    dev = torch.device("cuda", local_rank)
    _, N, H, C, seed, cu = WORKLOADS[args.config]
    P = world
    plan = U.ulysses_plan(N, H, 128, P, C, 0, 0, 0, cu)
    Nl = plan.rows_per_rank
    S = inputs.qkv_seq(N, H, P, C, seed, dev)
    shard = S[rank * Nl:(rank + 1) * Nl].clone()
    del S
    layer = peer.PeerLayer(plan) if args.transport == "peer" else peer.CollectiveLayer(plan)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        layer(shard)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize()
    sampler.begin()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        layer(shard)
    b.record(stream)
    torch.cuda.synchronize()
    sampler.end()
    dist.barrier()
    clocks = sampler.stop()
    if U.ulysses_last_device_error(plan) != 0:
        raise RuntimeError("a kernel reported a device error in the multi-GPU layer")
    ms = torch.tensor([a.elapsed_time(b) / args.steps], dtype=torch.float64, device=dev)
    dist.all_reduce(ms, op=dist.ReduceOp.MAX)
    ms = ms.item()
    del layer
    if rank != 0:
        return None
    flops = attn_flops(N, H, cu)
    per_rank = 3 if args.transport == "peer" else 2 + 2 * C   # launches (+ collectives) per rank per step
    return {
        "metric": "Ulysses layer µs; attn TFLOP/s and repack GB/s vs B200 peak",
        "value": round(ms * 1000.0, 2), "unit": "us per layer", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": False, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic N(0,1) bf16, seeded",
        "config": {"workload": f"{WORKLOAD_TEXT[args.config]}; split over {world} GPU(s), P = {world}",
                   "name": args.config, "P": P, "N": N, "Np": plan.padded_tokens,
                   "H": H, "D": 128, "planes": C, "seed": seed, "cu_seqlens": cu, "transport": args.transport,
                   "step": "one rank per GPU: push (or all-to-all) -> attention -> inverse exchange"},
        "attn_tflops_whole_job": round(flops / (ms * 1e-3) / 1e12, 1),
        "e2e": None, "gpu_launches": per_rank * args.steps, "clocks": clocks,
    }


def run_repack_stress(args, rank, world, local_rank):
    """Repack forward + backward at 250k tokens (QKVG), then a GB/s sweep over N."""
    import torch
    import torch.distributed as dist
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    P, N, H, C, seed, _ = WORKLOADS["stress250k"]
    stream = torch.cuda.current_stream()

    def time_pair(n, steps, warmup):
        plan = U.ulysses_plan(n, H, 128, P, C)
        Np = plan.padded_tokens
        S = inputs.qkv_seq(n, H, P, C, seed, dev)
        T = torch.empty((P, C, Np, H // P, 128), dtype=torch.bfloat16, device=dev)
        back = torch.empty_like(S)
        for _ in range(warmup):
            U.ulysses_repack_fwd(plan, S, T, stream)
            U.ulysses_repack_bwd(plan, T, back, C, stream)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        tf = tb = 0.0
        for _ in range(steps):
            ev[0].record(stream)
            U.ulysses_repack_fwd(plan, S, T, stream)
            ev[1].record(stream)
            U.ulysses_repack_bwd(plan, T, back, C, stream)
            ev[2].record(stream)
            torch.cuda.synchronize()
            tf += ev[0].elapsed_time(ev[1])
            tb += ev[1].elapsed_time(ev[2])
        ok = torch.equal(back, S)
        nbytes = 2 * S.numel() * 2          # read + write per direction
        return tf / steps, tb / steps, nbytes, ok, plan.plane_chunk

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    sampler.begin()
    tf, tb, nbytes, ok, chunk = time_pair(N, args.steps, args.warmup)
    sampler.end()
    clocks = sampler.stop()
    sweep = []
    for n in SWEEP_N:
        f, b, nb, ok_n, ch = time_pair(n, max(3, args.steps // 2), 3)
        sweep.append({"N": n, "fwd_gbs": round(nb / (f * 1e-3) / 1e9, 1), "bwd_gbs": round(nb / (b * 1e-3) / 1e9, 1),
                      "planes_per_launch": ch, "round_trip_exact": ok_n})
    if rank != 0:
        return None
    pk, pk_kind = peaks()
    gbs_f, gbs_b = nbytes / (tf * 1e-3) / 1e9, nbytes / (tb * 1e-3) / 1e9
    return {
        "metric": "Ulysses layer µs; attn TFLOP/s and repack GB/s vs B200 peak",
        "value": round((tf + tb) * 1000, 1), "unit": "us per repack fwd+bwd", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tf + tb, 3), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic N(0,1) bf16, seeded",
        "config": {"workload": WORKLOAD_TEXT["stress250k"], "name": "stress250k", "planes_per_launch": chunk,
                   "l2": "inputs larger than L2 (14.3 GB per direction)"},
        "repack_fwd_gbs": round(gbs_f, 1), "repack_bwd_gbs": round(gbs_b, 1), "round_trip_exact": ok,
        "roofline": {"bound": "hbm", "kernel": "repack_kernel", "achieved": round(gbs_f, 1), "peak": pk["hbm_gbs"],
                     "peak_kind": f"{pk_kind} copy", "unit": "GB/s", "frac": round(gbs_f / pk["hbm_gbs"], 3),
                     "frac_spec_8TBs": round(gbs_f / SPEC_PEAKS["hbm_gbs"], 3),
                     "traffic": recorded_traffic("repack_kernel", "stress250k")},
        "sweep": sweep, "clocks": clocks,
        "gpu_launches": 2 * C * args.steps,
    }


# ---------------------------------------------------------------------------- CPU oracle

def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# The oracle's sample of one layer, the same for ``cpu_baseline`` and for the
# ``--impl reference`` arm: attention of ORACLE_ROWS_PER_HEAD seeded query rows
# (all rows when N is smaller) of ORACLE_HEADS heads of rank 0 over all keys,
# and the repack of 1/ORACLE_TOKEN_FRAC of the tokens; each part extrapolated
# linearly (x N / rows x H / heads, x the token fraction).
ORACLE_ROWS_PER_HEAD = 4096
ORACLE_HEADS = 2
ORACLE_TOKEN_FRAC = 16


def oracle_sample(config, S_bits, rows_per_head=ORACLE_ROWS_PER_HEAD, heads=ORACLE_HEADS,
                  token_frac=ORACLE_TOKEN_FRAC):
    """Time the oracle on a bounded sample and extrapolate to one full layer (µs)."""
    import numpy as np
    from oracle import ulysses_oracle as orc
    P, N, H, C, seed, cu = WORKLOADS[config]
    Np = S_bits.shape[0]
    Hl = H // P
    if config == "stress250k":   # repack forward + backward of all planes only
        ns = max(P, (Np // token_frac) // P * P)
        t0 = time.perf_counter()
        Tsub = orc.repack_fwd(np.ascontiguousarray(S_bits[:ns]), P)
        orc.repack_bwd(Tsub)
        t = (time.perf_counter() - t0) * (Np / ns)
        return t * 1e6, f"repack fwd+bwd of {ns}/{Np} tokens (x{Np / ns:.1f}), extrapolated linearly"
    # repack: a token slice (multiple of P rows), scaled by the slice fraction
    ns = max(P, (Np // token_frac) // P * P)
    t0 = time.perf_counter()
    Tsub = orc.repack_fwd(np.ascontiguousarray(S_bits[:ns]), P)
    t_rf = (time.perf_counter() - t0) * (Np / ns)
    t0 = time.perf_counter()
    orc.repack_bwd(Tsub[:, :1])
    t_rb = (time.perf_counter() - t0) * (Np / ns)
    # attention: `heads` heads of rank 0 (every head when N is small enough for
    # all rows), `rows_per_head` sampled rows, all keys
    if N <= rows_per_head:
        heads = H // P
    heads = min(heads, H // P)
    T = np.empty((1, 3, Np, heads, 128), dtype=np.uint16)
    for c in range(3):
        T[0, c] = S_bits[:, c, :heads, :]
    rows = orc.sample_rows(N, rows_per_head, seed, cu)
    t0 = time.perf_counter()
    orc.attention_heads(T, N, 1.0 / math.sqrt(128), cu_seqlens=cu, rows=rows)
    t_at = (time.perf_counter() - t0) * (N / rows.size) * (H / heads)
    total_us = (t_rf + t_at + t_rb) * 1e6
    sample = (f"repack of {ns}/{Np} tokens (x{Np / ns:.1f}); attention of {rows.size} query rows x {heads} heads "
              f"over all keys (x{N / rows.size:.2f} rows x {H / heads:.1f} heads = x{(N / rows.size) * (H / heads):.1f});"
              f" extrapolated linearly to one layer")
    return total_us, sample


def cpu_baseline(config, S):
    from ulysses_sequence_attention_repack_b200 import inputs
    S_bits = inputs.host_bits(S)
    us, sample = oracle_sample(config, S_bits)
    return {"value": round(us, 1), "unit": "us per layer", "cores": _cores(), "kind": "oracle",
            "sample": sample}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, rank 0 only, on a bounded sample per step."""
    if rank != 0:
        return None
    import numpy as np
    import torch
    P, N, H, C, seed, cu = WORKLOADS[args.config]
    sys.path.insert(0, ROOT)
    from ulysses_sequence_attention_repack_b200 import inputs
    S = inputs.qkv_seq(N, H, P, C, seed, "cpu")
    S_bits = inputs.host_bits(S)
    del S
    for _ in range(args.warmup):
        oracle_sample(args.config, S_bits)
    vals, sample = [], ""
    t_start = time.perf_counter()
    for _ in range(args.steps):
        v, sample = oracle_sample(args.config, S_bits)
        vals.append(v)
    wall = time.perf_counter() - t_start
    value = statistics.mean(vals)
    return {
        "impl": "reference",
        "metric": "Ulysses layer µs; attn TFLOP/s and repack GB/s vs B200 peak",
        "value": round(value, 1), "unit": "us per layer", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(value / 1000, 3), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic N(0,1) bf16, seeded",
        "config": {"workload": WORKLOAD_TEXT[args.config], "name": args.config},
        "cpu_baseline": {"value": round(value, 1), "unit": "us per layer", "cores": _cores(), "kind": "oracle",
                         "sample": sample, "wall_s": round(wall, 1)},
        "e2e": {"value": round(value, 1), "unit": "us per layer", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "numpy": np.__version__, "torch": torch.__version__,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="long104k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the other layer workloads timed after the main one")
    ap.add_argument("--pair-attention", action="store_true",
                    help="run the bf16 attention on CTA pairs (ULYSSES_PLAN_PAIR_ATTENTION) instead of one CTA per SM")
    ap.add_argument("--transport", default="replicas", choices=["replicas", "peer", "nccl"],
                    help="replicas (default): every GPU runs the whole one-GPU layer; peer / nccl: "
                         "the layer split across the launched GPUs, one rank each")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    multi = args.transport != "replicas"
    if multi and (args.config in FP8 or args.config in CAUSAL or args.config == "stress250k"):
        ap.error("--transport peer|nccl runs the bf16 non-causal layer configs")
    if world > 1 or multi:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        if world == 1:   # a one-rank group of its own
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            if "MASTER_PORT" not in os.environ:
                import socket
                with socket.socket() as sk:
                    sk.bind(("127.0.0.1", 0))
                    os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if multi:
            line = run_transport(args, rank, world, local_rank)
        elif args.config == "stress250k":
            line = run_repack_stress(args, rank, world, local_rank)
        elif args.config in FP8:
            line = run_fp8(args, rank, world, local_rank)
        else:
            line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 or multi:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
