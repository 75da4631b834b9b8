#!/usr/bin/env python
"""Benchmark of the LLSA training step (forward + backward of the attention op).

One step = the whole hot path on one batch of device-resident synthetic input:
pyramid -> hierarchical selection -> attention forward -> index transpose -> attention
backward (five C-ABI calls, 12 kernel launches at the default workload).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload headline-65536]

Multi-GPU runs (torchrun, one process per GPU) are weak-scaled independent replicas: every
rank runs the whole workload on its own GPU, with no data-path collective; the step time is
the maximum over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
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

METRIC = "LLSA fwd+bwd tokens/sec at N=65536 bf16, 1 B200; % of roofline"
UNIT = "tokens/s"
KERNELS_PER_STEP_HINT = 16


# ----------------------------------------------------------------------------- distributed

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world, local, backend: str = "nccl"):
    import torch
    import torch.distributed as dist
    if world > 1:
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_max(x: float, world: int, device: str = "cuda") -> float:
    """Maximum of x over all ranks (the step time of a multi-GPU run is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_step: int, steps: int, world: int, ms_total: float) -> float:
    """Whole-job tokens/s: every rank runs `steps` steps of its own replica."""
    return world * steps * tokens_per_step / (ms_total / 1000.0)


def dist_done(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons while running."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_uuid: str):
        self.uuid = gpu_uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self, load_threshold_w: float = 250.0) -> dict:
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r[2] >= load_threshold_w] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows)}


# ----------------------------------------------------------------------------- algorithmic counts

def workload_counts(cfg, pairs_l1: int, all_top: bool = False, select_launches: int | None = None):
    """Algorithmic bytes and FLOPs per launch of each kernel for one step of ``cfg``.

    Per query block the forward gathers the KV list (T tokens x 64 channels x 2 bytes for K
    and for V) and streams Q, O and LSE; the query-major backward gathers the same list and
    streams Q, dO, O, dQ, LSE and Delta; the key-major backward streams K_j, V_j, dK_j, dV_j
    per fine key block and Q, dO, LSE, Delta per (key block, query block) pair.  FLOPs are
    4*16*T*64 per block (forward), 6*16*T*64 (query-major backward: S, dP, dQ) and
    8*16*16*64 per pair (key-major backward: S, dP, dV, dK).
    """
    D, e = cfg.D, 2
    bh = cfg.B * cfg.H
    n = cfg.level_sizes()
    n1 = n[1]
    coarse = coarse_entries(cfg, all_top)
    T = 16 * cfg.topk + coarse
    blocks = bh * n1
    tile = 16 * D * e
    row_stream = 16 * 4
    counts = {
        "attn_fwd_bf16": dict(bytes=blocks * (T * D * e * 2 + 2 * tile + row_stream),
                              flops=4 * blocks * 16 * T * D),
        "attn_bwd_dq_bf16": dict(bytes=blocks * (T * D * e * 2 + 4 * tile + 2 * row_stream),
                                 flops=6 * blocks * 16 * T * D),
        "attn_bwd_dkdv_bf16": dict(bytes=blocks * 4 * tile + pairs_l1 * (2 * tile + 2 * row_stream),
                                   flops=8 * pairs_l1 * 16 * 16 * D),
        "pyramid_l12": dict(bytes=3 * (bh * cfg.N * D * e + bh * (n1 + (n[2] if cfg.levels >= 2 else 0)) * D * 4),
                            flops=0),
    }
    L, K = cfg.levels, cfg.topk
    f4 = 4
    # selection, all levels of a step (its launches share the name "select"): the coarsest
    # level reads its q and k rows (plus, pooled in the same launch, levels >= 3 read from the
    # level below); a finer level l reads, per parent group, the 16K candidate rows once and
    # the 16 query rows, and writes the indices.
    sel_bytes = 2 * bh * n[L] * D * f4 + bh * n[L] * K * 4
    sel_flops = 2 * bh * n[L] * n[L] * D
    for lev in range(3, L + 1):
        sel_bytes += 3 * (bh * n[lev - 1] * D * f4 + bh * n[lev] * D * f4)
    for lev in range(L - 1, 0, -1):
        groups = bh * n[lev + 1]
        sel_bytes += groups * (16 * K * D * f4 + 16 * D * f4 + K * 4) + bh * n[lev] * K * 4
        sel_flops += 2 * bh * n[lev] * 16 * K * D
    # per launch: the step's selection work over its selection launches (L, or L - 1 when the
    # level-2 selection runs inside the level-1 launch)
    nsel = select_launches or L
    counts["select"] = dict(bytes=sel_bytes // nsel, flops=sel_flops // nsel)
    # transpose: E entries over all levels; hist reads idx, scatter reads idx and writes the
    # bucketed entries, bucket reads them and writes col and row_ptr
    entries = sum(bh * n[lev] * K for lev in range(1, L + 1))
    rows = sum(bh * (n[lev] + 1) for lev in range(1, L + 1))
    counts["transpose_hist"] = dict(bytes=entries * 4, flops=0)
    counts["transpose_scatter"] = dict(bytes=2 * entries * 4, flops=0)
    counts["transpose_bucket"] = dict(bytes=2 * entries * 4 + rows * 4, flops=0)
    counts["dkdv_order_count"] = dict(bytes=bh * (n1 + 1) * 4, flops=0)
    counts["dkdv_order_scatter"] = dict(bytes=bh * (n1 + 1) * 4 + bh * n1 * 16, flops=0)
    if L >= 2:
        ctas = bh * n[2] * ((coarse + 15) // 16)
        # per (level-2 group, coarse tile): 16 query blocks' Q, dO, LSE, Delta, the coarse K/V
        # rows (fp32), the fp32 partials written
        counts["attn_bwd_coarse_bf16"] = dict(
            bytes=ctas * (16 * (2 * tile + 2 * row_stream) + 2 * 16 * D * f4) + 2 * bh * n[2] * coarse * D * f4,
            flops=8 * ctas * 16 * 16 * 16 * D)
        cg_rows = sum(bh * n[lev] for lev in range(2, L + 1))
        counts["coarse_grad_reduce"] = dict(bytes=2 * bh * n[2] * coarse * D * f4 + 2 * cg_rows * D * f4, flops=0)
    return counts


def coarse_entries(cfg, all_top: bool = False) -> int:
    """Coarse KV entries per query block: (L-1) K, or (L-2) K + n_L for the all-coarsest variant."""
    L, K = cfg.levels, cfg.topk
    if L < 2:
        return 0
    return (L - 2) * K + cfg.level_sizes()[L] if all_top else (L - 1) * K


def enrichment(args) -> dict:
    """Keyword arguments of the enrichment variants chosen on the command line."""
    return dict(log_bias=args.log_bias, all_top=args.all_top, level1=args.level1)


def enrichment_text(args) -> str:
    parts = ["log-count bias ln(16^l) on coarse scores" if args.log_bias else "unit weight"]
    if args.all_top:
        parts.append("all n_L coarsest tokens in every list")
    if args.level1:
        parts.append("level-1 pooled token of every selected block (folded into its fine tile)")
    return "; ".join(parts)


# ----------------------------------------------------------------------------- oracle sample

def oracle_sample(cfg, inputs, heads: int, nblocks: int | None, log_bias: bool = False, all_top: bool = False,
                  level1: bool = False):
    """Time the CPU oracle on ``heads`` (b=0) heads of the workload: pyramid, selection and
    transpose for each whole head, forward and backward for ``nblocks`` query blocks per
    head (all blocks if None).  Returns (tokens/s extrapolated to the full workload, dict)."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    from oracle import llsa_oracle as orc
    from synthetic import to_f32_numpy, to_f64_numpy

    n1 = cfg.N // 16
    blocks = None if nblocks is None or nblocks >= n1 else np.linspace(0, n1 - 1, nblocks).astype(np.int64)
    nb = n1 if blocks is None else len(blocks)
    t_fixed = t_attn = 0.0
    with threadpool_limits(1):
        for h in range(heads):
            sl = (slice(0, 1), slice(h, h + 1))
            q32, k32, v32 = (to_f32_numpy(inputs[x][sl]) for x in ("q", "k", "v"))
            q, k, v, do = (to_f64_numpy(inputs[x][sl]) for x in ("q", "k", "v", "do"))
            t0 = time.perf_counter()
            qp, kp, vp = (orc.build_pyramid(a, cfg.levels) for a in (q32, k32, v32))
            idx = orc.select(qp, kp, cfg.topk)
            orc.index_transpose_all(idx)
            t1 = time.perf_counter()
            o, lse = orc.forward(q, k, v, kp, vp, idx, blocks=blocks, log_bias=log_bias, all_top=all_top,
                                 level1=level1)
            if cfg.backward:
                orc.backward(q, k, v, o, lse, do, kp, vp, idx, blocks=blocks, log_bias=log_bias, all_top=all_top,
                             level1=level1)
            t2 = time.perf_counter()
            t_fixed += t1 - t0
            t_attn += t2 - t1
    # per head: fixed part + attention scaled from nb sampled blocks to all n1 blocks
    per_head = (t_fixed + t_attn * (n1 / nb)) / heads
    full_step = per_head * cfg.B * cfg.H
    info = {"heads": heads, "blocks_per_head": nb, "seconds": t_fixed + t_attn, "t_full_step_est_s": full_step,
            "t_fixed_per_head": t_fixed / heads, "t_attn_per_block": t_attn / (heads * nb)}
    return cfg.B * cfg.N / full_step, info


# ----------------------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.nn.functional as F

    from log_linear_hierarchical_b200 import api
    from synthetic import WORKLOADS, make_config_inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dist_init(world, local)
    cfg = WORKLOADS[args.workload]
    dtype = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    host = make_config_inputs(cfg, with_do=True)
    pinned = {k: v.pin_memory() for k, v in host.items()}
    dev = {k: v.cuda(non_blocking=True) for k, v in pinned.items()}
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, dtype, **enrichment(args))
    buf = api.LLSABuffers.allocate(shape, "cuda", dtype)
    stream = torch.cuda.current_stream()

    def step():
        api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = api.llsa_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    # one traced step to size the trace of the timed region
    probe = api.LaunchTrace(64)
    with probe:
        step()
    per_step = probe.used
    torch.cuda.synchronize()

    # The timed region is one launch of a plan: the K steps captured into one CUDA graph
    # (transpose on a second stream, kernels chained by programmatic dependent launch).
    # The plan is built and launched once before timing (graph upload).  Per-kernel times
    # come from a second plan of the same K steps captured with trace events around every
    # kernel, launched after the timed region (event nodes between kernels turn the
    # programmatic edges into full ones, so it runs slightly slower than the timed plan).
    plan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=args.steps)
    plan.launch(stream)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(local)
    sampler = ClockSampler("GPU-" + str(props.uuid)) if rank == 0 or world == 1 else None
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.start()
    dist_barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    plan.launch(stream)
    end.record(stream)
    torch.cuda.synchronize()
    dist_barrier(world)
    if sampler:
        sampler.stop()
    ms_local = start.elapsed_time(end)
    ms_total = dist_max(ms_local, world)
    status = api.llsa_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    plan.close()

    # the traced plan: same steps, trace events recorded by the graph at every kernel
    trace = api.LaunchTrace(per_step * args.steps)
    with trace:
        tplan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=args.steps)
    tplan.launch(stream)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(world)
    t0.record(stream)
    tplan.launch(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    traced_ms_per_step = dist_max(t0.elapsed_time(t1), world) / args.steps

    # per-kernel averages over the timed region
    launches = trace.launches()
    per_kernel: dict[str, list[float]] = {}
    for name, ms in launches:
        per_kernel.setdefault(name, []).append(ms)
    kern = {k: {"launches": len(v), "avg_us": 1000 * sum(v) / len(v), "total_ms": sum(v)} for k, v in per_kernel.items()}
    total_kernel_ms = sum(x["total_ms"] for x in kern.values())
    for x in kern.values():
        x["share"] = x["total_ms"] / total_kernel_ms

    tokens_per_step = cfg.B * cfg.N
    value = weak_scaling_value(tokens_per_step, args.steps, world, ms_total)
    ms_per_step = ms_total / args.steps

    # algorithmic roofline of the dominant kernel
    rps, _ = buf.csr_levels()
    pairs_l1 = int(rps[0][..., -1].sum().item())
    sel_launches = round(kern["select"]["launches"] / args.steps) if "select" in kern else None
    counts = workload_counts(cfg, pairs_l1, args.all_top, sel_launches)
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else None
    hbm_peak = peaks["hbm_gbs"] if peaks else 6650.0
    tensor_peak = peaks["bf16_tflops_sustained"] if peaks else 1400.0
    dominant = max(kern, key=lambda k: kern[k]["total_ms"])
    roofline = None
    if dominant in counts:
        c = counts[dominant]
        sec = kern[dominant]["avg_us"] * 1e-6
        achieved = c["bytes"] / sec / 1e9
        roofline = {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                    "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                    "traffic": traffic_per_launch(dominant, cfg),
                    "peak_source": "measured" if peaks else "fallback",
                    "algorithmic_bytes_per_launch": c["bytes"],
                    "tensor_achieved_tflops": round(c["flops"] / sec / 1e12, 2),
                    "tensor_frac_of_sustained_bf16": round(c["flops"] / sec / 1e12 / tensor_peak, 4)}
    kernels_roof = {}
    for k, c in counts.items():
        if k in kern:
            sec = kern[k]["avg_us"] * 1e-6
            kernels_roof[k] = {"avg_us": round(kern[k]["avg_us"], 2), "share": round(kern[k]["share"], 4),
                               "hbm_frac": round(c["bytes"] / sec / 1e9 / hbm_peak, 4),
                               "tensor_frac": round(c["flops"] / sec / 1e12 / tensor_peak, 4) if c["flops"] else 0.0}
    # whole-step roofline as the workload defines it: the slower of the selected attention's
    # FLOPs at the bf16 tensor peak and its modelled bytes (gathers and pyramid) at the HBM
    # peak; the other kernels have their own fractions in `kernels`
    step_kernels = ("attn_fwd_bf16", "attn_bwd_dq_bf16", "attn_bwd_dkdv_bf16", "pyramid_l12")
    step_bytes = sum(c["bytes"] for k, c in counts.items() if k in kern and k in step_kernels)
    step_flops = sum(c["flops"] for k, c in counts.items() if k in kern and k in step_kernels)
    step_roof_ms = 1000 * max(step_bytes / (hbm_peak * 1e9), step_flops / (tensor_peak * 1e12))

    # end to end through the public API with host buffers, as a training loop feeds it: two
    # device buffer sets, each with its own one-step plan; step i's inputs are copied in on
    # an upload stream while step i-1 computes, and step i's results are copied out on a
    # download stream while step i+1 computes.  Every step's inputs and results cross the
    # host link inside the timed region; the two directions and the compute overlap.
    tplan.close()
    e2e_steps = max(2, min(args.steps, 20))
    host_out = [{k: torch.empty(cfg.B, cfg.H, cfg.N, cfg.D, dtype=dtype).pin_memory() for k in ("o", "dq", "dk", "dv")}
                for _ in range(2)]
    sets = []
    for si in range(2):
        d_in = dev if si == 0 else {k: torch.empty_like(v) for k, v in dev.items()}
        b = buf if si == 0 else api.LLSABuffers.allocate(shape, "cuda", dtype)
        sets.append((d_in, b, api.LLSAPlan(shape, d_in["q"], d_in["k"], d_in["v"], d_in["do"], b, repeat=1)))
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    computed = [torch.cuda.Event() for _ in range(2)]   # set s: its plan has run (inputs free)
    drained = [torch.cuda.Event() for _ in range(2)]    # set s: its results are on the host
    for si in range(2):
        computed[si].record(stream)
        drained[si].record(stream)
    in_bytes = sum(t.numel() * t.element_size() for t in pinned.values())
    out_bytes = sum(t.numel() * t.element_size() for t in host_out[0].values())
    dist_barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_stream(stream)
    for i in range(e2e_steps):
        si = i % 2
        d_in, b, plan_s = sets[si]
        loaded = torch.cuda.Event()
        with torch.cuda.stream(up):
            up.wait_event(computed[si])
            for k in ("q", "k", "v", "do"):
                d_in[k].copy_(pinned[k], non_blocking=True)
            loaded.record(up)
        stream.wait_event(loaded)
        stream.wait_event(drained[si])
        plan_s.launch(stream)
        computed[si].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed[si])
            for k in ("o", "dq", "dk", "dv"):
                host_out[si][k].copy_(getattr(b, k), non_blocking=True)
            drained[si].record(down)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dist_max(e0.elapsed_time(e1), world)
    for _, _, plan_s in sets:
        plan_s.close()
    last = (e2e_steps - 1) % 2
    assert torch.equal(host_out[last]["dk"], sets[last][1].dk.cpu()), "the downloaded result differs from the device's"
    e2e_value = world * e2e_steps * tokens_per_step / (e2e_ms / 1000.0)

    # quadtree token order (llsa_token_permute) of one input tensor: HBM streaming
    zperm = None
    side_ok = (cfg.N & (cfg.N - 1)) == 0 and int(round(cfg.N ** 0.5)) ** 2 == cfg.N
    if side_ok:
        zdst = torch.empty_like(dev["q"])
        for _ in range(3):
            api.llsa_token_permute(shape, dev["q"], zdst, to_z_order=True, stream=stream)
        torch.cuda.synchronize()
        z0, z1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        zreps = 20
        z0.record(stream)
        for _ in range(zreps):
            api.llsa_token_permute(shape, dev["q"], zdst, to_z_order=True, stream=stream)
        z1.record(stream)
        torch.cuda.synchronize()
        zus = 1000 * z0.elapsed_time(z1) / zreps
        zbytes = 2 * dev["q"].numel() * dev["q"].element_size()
        zperm = {"tensor": "q to Z order", "avg_us": round(zus, 2), "bytes": zbytes,
                 "gbs": round(zbytes / (zus * 1e-6) / 1e9, 1), "hbm_frac": round(zbytes / (zus * 1e-6) / 1e9 / hbm_peak, 4)}
        del zdst

    # dense attention at the same shape (torch SDPA, flash backend), forward + backward
    dense = None
    if world == 1:
        q = dev["q"].detach().clone().requires_grad_(True)
        k = dev["k"].detach().clone().requires_grad_(True)
        v = dev["v"].detach().clone().requires_grad_(True)
        for _ in range(2):
            F.scaled_dot_product_attention(q, k, v).backward(dev["do"])
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        d0.record(stream)
        for _ in range(reps):
            F.scaled_dot_product_attention(q, k, v).backward(dev["do"])
        d1.record(stream)
        torch.cuda.synchronize()
        dms = d0.elapsed_time(d1) / reps
        dense = {"impl": "torch scaled_dot_product_attention (bf16, non-causal), forward + backward",
                 "ms_per_step": round(dms, 3), "tokens_per_s": round(tokens_per_step / (dms / 1000.0), 1),
                 "llsa_speedup": round(dms / ms_per_step, 2)}
        del q, k, v

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, info = oracle_sample(cfg, host, heads=2, nblocks=None, **enrichment(args))
        cpu = {"value": round(val, 2), "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": (f"numpy fp64 oracle, 1 thread: pyramid, selection, transpose, forward and backward of "
                          f"heads (b=0, h=0..1), {info['seconds']:.1f} s, extrapolated to {cfg.B * cfg.H} heads")}

    clocks = sampler.summary() if sampler else None
    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == "bf16" else "f32",
        "data": "synthetic (seeded smooth-field Q/K in Z order, N(0,1) V and dO)",
        "config": {"workload": f"{cfg.name}: {cfg.describe()}", "B": cfg.B, "H": cfg.H, "N": cfg.N, "D": cfg.D,
                   "block": cfg.block, "levels": cfg.levels, "topk": cfg.topk,
                   "kv_len": 16 * cfg.topk + (cfg.topk if args.level1 else 0) + coarse_entries(cfg, args.all_top),
                   "step": "pyramid + select + forward + index transpose + backward",
                   "enrichment": enrichment_text(args),
                   "launch": ("K steps as one CUDA graph (llsa_plan_create repeat=K), kernels chained by "
                              "programmatic dependent launch; transpose on a second stream"),
                   "kernel_times_from": ("a second plan of the same K steps with trace events around every "
                                         f"kernel, launched after the timed one: {traced_ms_per_step:.4f} ms per step"),
                   "parallelism": f"dp{world}: independent replicas, no collective",
                   "l2": "inputs larger than L2: q, k, v, dO are 201 MB per replica vs 126 MB L2; no flush"},
        "roofline": roofline,
        "step_roofline": {"modelled_bytes": step_bytes, "flops": step_flops, "roofline_ms": round(step_roof_ms, 4),
                          "frac": round(step_roof_ms / ms_per_step, 4)},
        "kernels": kernels_roof,
        "kernel_times": {k: {"launches": v["launches"], "avg_us": round(v["avg_us"], 2), "share": round(v["share"], 4)}
                         for k, v in sorted(kern.items(), key=lambda kv: -kv[1]["total_ms"])},
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": out_bytes, "steps": e2e_steps,
                "api": ("log_linear_hierarchical_b200.LLSAPlan (one captured step, llsa_plan_launch) on two "
                        "device buffer sets; each step's inputs copied in from pinned host memory on an upload "
                        "stream and its results copied out on a download stream, overlapping the neighbouring "
                        "steps")},
        "dense_attention": dense,
        "token_permute": zperm,
        "gpu_launches": trace.used,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    del trace
    dist_done(world)


def traffic_per_launch(kernel: str, cfg):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel sources (profiles/ncu_traffic.txt lines: kernel workload bytes source-hash)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    h = source_hash()
    for ln in open(path):
        parts = ln.split()
        if len(parts) == 4 and parts[0] == kernel and parts[1] == cfg.name and parts[3] == h:
            return float(parts[2])
    return None


def source_hash() -> str:
    import hashlib
    d = os.path.join(ROOT, "log_linear_hierarchical_b200", "csrc")
    m = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f.endswith(".cuh"):  # every kernel and its launch-shaping constants live in the headers
            m.update(open(os.path.join(d, f), "rb").read())
    return m.hexdigest()[:12]


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The CPU oracle as the reference arm: rank 0 only, each step a bounded sample."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from synthetic import WORKLOADS, make_config_inputs

    cfg = WORKLOADS[args.workload]
    host = make_config_inputs(cfg, with_do=True)
    n1 = cfg.N // 16
    # size each step's sample so that warm-up + steps stay near two minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    _, probe = oracle_sample(cfg, host, heads=1, nblocks=16, **enrichment(args))
    per_block = max(1e-6, probe["t_attn_per_block"])
    nblocks = int(max(16, min(n1, (budget - probe["t_fixed_per_head"]) / per_block)))
    for _ in range(args.warmup):
        oracle_sample(cfg, host, heads=1, nblocks=nblocks, **enrichment(args))
    vals, secs = [], 0.0
    for _ in range(args.steps):
        v, info = oracle_sample(cfg, host, heads=1, nblocks=nblocks, **enrichment(args))
        vals.append(v)
        secs += info["seconds"]
    value = statistics.median(vals)
    tokens_per_step = cfg.B * cfg.N
    ms_per_step = 1000.0 * tokens_per_step / value
    sample = (f"numpy fp64 oracle, 1 thread, per step: pyramid, selection and transpose of head (b=0, h=0) and "
              f"forward+backward of {nblocks} of its {n1} query blocks, extrapolated to all blocks and "
              f"{cfg.B * cfg.H} heads; median over {args.steps} steps")
    result = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": {"workload": f"{cfg.name}: {cfg.describe()}", "B": cfg.B, "H": cfg.H, "N": cfg.N, "D": cfg.D,
                   "block": cfg.block, "levels": cfg.levels, "topk": cfg.topk,
                   "kv_len": 16 * cfg.topk + (cfg.topk if args.level1 else 0) + coarse_entries(cfg, args.all_top),
                   "enrichment": enrichment_text(args)},
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def run_profile(args):
    """Only the timed step, for profilers: W warm-up steps then K steps, one line of output."""
    import torch

    from log_linear_hierarchical_b200 import api
    from synthetic import WORKLOADS, make_config_inputs

    cfg = WORKLOADS[args.workload]
    dtype = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    dev = {k: v.cuda() for k, v in make_config_inputs(cfg, with_do=True).items()}
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, dtype, **enrichment(args))
    buf = api.LLSABuffers.allocate(shape, "cuda", dtype)
    for _ in range(args.warmup + args.steps):
        api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    torch.cuda.synchronize()
    status = api.llsa_device_status()
    print(json.dumps({"profile_run": cfg.name, "steps": args.steps, "warmup": args.warmup, "status": status}))
    if status != 0:
        sys.exit(1)


def _workload_names():
    from synthetic import WORKLOADS
    return WORKLOADS.keys()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="headline-65536", choices=list(_workload_names()),
                    help="synthetic workload (default: the headline N=65536 step)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle sample")
    ap.add_argument("--profile", action="store_true", help="run only the steps (for ncu), print no metric")
    ap.add_argument("--log-bias", action="store_true",
                    help="the log-count enrichment variant (ln 16^l on level-l coarse scores)")
    ap.add_argument("--all-top", action="store_true",
                    help="the all-coarsest enrichment variant (every level-L token in every list)")
    ap.add_argument("--level1", action="store_true",
                    help="the level-1 enrichment variant (each selected block's mean token in the list)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
