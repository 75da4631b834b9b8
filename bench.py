#!/usr/bin/env python
"""Benchmark of the LLSA training step (forward + backward of the attention op).

One step = the whole hot path on one batch of device-resident synthetic input:
pyramid -> hierarchical selection -> attention forward -> index transpose -> attention
backward (the five C-ABI calls as one llsa_train_step; 15 kernel launches at the default
workload, counted live in `gpu_launches`).

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
    # the pyramid and every selection level in one launch (bf16, small coarsest level)
    counts["pyramid_select"] = dict(bytes=counts["pyramid_l12"]["bytes"] + sel_bytes, flops=sel_flops)
    # transpose: E entries over all levels; hist reads idx, scatter reads idx and writes the
    # bucketed entries, bucket reads them and writes col and row_ptr
    entries = sum(bh * n[lev] * K for lev in range(1, L + 1))
    rows = sum(bh * (n[lev] + 1) for lev in range(1, L + 1))
    counts["transpose_hist"] = dict(bytes=entries * 4, flops=0)
    counts["transpose_scatter"] = dict(bytes=2 * entries * 4, flops=0)
    counts["transpose_bucket"] = dict(bytes=2 * entries * 4 + rows * 4, flops=0)
    hist = 0   # the scan reads and rewrites every (bucket, tile) count of every problem
    for lev in range(1, L + 1):
        width = 1
        while -(-n[lev] // width) > 64:
            width *= 2
        hist += bh * (-(-n[lev] // width) * -(-(n[lev] * K) // 4096) + 1)
    counts["transpose_scan"] = dict(bytes=2 * hist * 4, flops=0)
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


def compulsory_bytes(cfg, elem: int) -> int:
    """DRAM bytes no implementation of the step can avoid: q, k, v, dO read once; o, dq, dk,
    dv and LSE written once; the pyramids, the selection and its CSR written once."""
    bh = cfg.B * cfg.H
    n = cfg.level_sizes()
    L, K, D = cfg.levels, cfg.topk, cfg.D
    act = 8 * bh * cfg.N * D * elem
    lse = bh * cfg.N * 4
    pyr = 3 * sum(bh * n[lev] * D * 4 for lev in range(1, L + 1))
    sel = 2 * sum(bh * n[lev] * K * 4 for lev in range(1, L + 1)) + sum(bh * (n[lev] + 1) * 4 for lev in range(1, L + 1))
    return act + lse + pyr + sel


def measure_gather_peak(api, torch, stream, sms: int) -> dict:
    """L2 -> SM gather ceiling: llsa_gather_probe (the attention kernels' 16 x 64 bf16 TMA tile
    gather and nothing else) over random tiles of a 32 MiB buffer that stays in L2; the best
    bytes per second over ring depths and CTAs per SM."""
    rows = 1 << 18
    gen = torch.Generator().manual_seed(11)
    src = torch.randn(rows, 64, generator=gen).to(torch.bfloat16).cuda()
    ntiles = 1 << 19
    tile_rows = (torch.randint(0, rows // 16, (ntiles,), generator=gen) * 16).to(torch.int32).cuda()
    best = {"gbs": 0.0}
    for stages in (2, 4, 8):
        for per_sm in (2, 4, 8):
            ctas = sms * per_sm
            api.llsa_gather_probe(src, tile_rows, stages, ctas, stream)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 3
            e0.record(stream)
            for _ in range(reps):
                api.llsa_gather_probe(src, tile_rows, stages, ctas, stream)
            e1.record(stream)
            torch.cuda.synchronize()
            gbs = reps * ntiles * 2048 / (e0.elapsed_time(e1) * 1e-3) / 1e9
            if gbs > best["gbs"]:
                best = {"gbs": round(gbs, 1), "stages": stages, "ctas": ctas}
    best.update(buffer_mib=rows * 128 >> 20, tile_bytes=2048, tiles_per_launch=ntiles)
    return best


def run_probe(args):
    """Only the L2 gather ceiling (llsa_gather_probe sweep), one JSON line: for profilers."""
    import torch

    from log_linear_hierarchical_b200 import api
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    best = measure_gather_peak(api, torch, torch.cuda.current_stream(), sms)
    print(json.dumps({"gather_probe": best}))


def enrichment(args) -> dict:
    """Keyword arguments of the enrichment variants chosen on the command line."""
    return dict(log_bias=args.log_bias, all_top=args.all_top, level1=args.level1)


def to_grid_order(host: dict, cfg) -> dict:
    """The synthetic tokens (generated in quadtree order) moved to the row-major order of the
    square grid: what a caller that passes LLSA_FLAG_GRID_ORDER hands the library."""
    import torch
    from synthetic import morton_order
    perm = torch.from_numpy(morton_order(cfg.grid))   # raster position of each Z position
    return {k: torch.empty_like(v).index_copy_(2, perm, v) for k, v in host.items()}


def enrichment_text(args) -> str:
    parts = ["log-count bias ln(16^l) on coarse scores" if args.log_bias else "unit weight"]
    if args.all_top:
        parts.append("all n_L coarsest tokens in every list")
    if args.level1:
        parts.append("level-1 pooled token of every selected block (folded into its fine tile)")
    return "; ".join(parts)


# ----------------------------------------------------------------------------- oracle on host cores
# The CPU baseline and the reference arm run the oracle, as it stands, on every host core: a
# pool of worker processes (spawn start method) over (head, query-block chunk).  Inputs live
# in shared memory (fp32, the exact values of the device inputs); each task writes its query
# blocks' O, LSE and dQ rows in place and adds its dK/dV contribution to its head's shared
# fp64 accumulator under that head's lock.  A step is: per head, pyramid + selection + index
# transpose; then per (head, chunk), forward + backward of the chunk's query blocks.

_ORC = {}


def _orc_attach(names, shape, flags, levels, topk, locks):
    """Worker initializer: map the shared inputs and outputs, one BLAS thread per process."""
    import numpy as np
    from multiprocessing import shared_memory
    from threadpoolctl import threadpool_limits

    threadpool_limits(1)
    _ORC["shm"] = {k: shared_memory.SharedMemory(name=v) for k, v in names.items()}
    B, H, N, D = shape
    for k, m in _ORC["shm"].items():
        if k in ("q", "k", "v", "do"):
            _ORC[k] = np.ndarray((B, H, N, D), dtype=np.float32, buffer=m.buf)
        elif k == "lse":
            _ORC[k] = np.ndarray((B, H, N), dtype=np.float64, buffer=m.buf)
        else:
            _ORC[k] = np.ndarray((B, H, N, D), dtype=np.float64, buffer=m.buf)
    _ORC.update(flags=flags, levels=levels, topk=topk, locks=locks)


def _orc_head(bh):
    """Pyramid, selection and index transpose of one head; returns what the chunks need."""
    from oracle import llsa_oracle as orc
    b, h = bh
    sl = (slice(b, b + 1), slice(h, h + 1))
    qp, kp, vp = (orc.build_pyramid(_ORC[x][sl], _ORC["levels"]) for x in ("q", "k", "v"))
    idx = orc.select(qp, kp, _ORC["topk"])
    orc.index_transpose_all(idx)
    return kp, vp, idx


def _orc_chunk(task):
    """Forward and backward of one chunk of query blocks of one head."""
    import numpy as np
    from oracle import llsa_oracle as orc
    (b, h), blocks, kp, vp, idx, head_no, backward = task
    sl = (slice(b, b + 1), slice(h, h + 1))
    q, k, v = (_ORC[x][sl].astype(np.float64) for x in ("q", "k", "v"))
    o, lse = orc.forward(q, k, v, kp, vp, idx, blocks=blocks, **_ORC["flags"])
    rows = (blocks[:, None] * 16 + np.arange(16)).ravel()
    _ORC["o"][b, h, rows] = o[0, 0, rows]
    _ORC["lse"][b, h, rows] = lse[0, 0, rows]
    if backward:
        do = _ORC["do"][sl].astype(np.float64)
        dq, dk, dv = orc.backward(q, k, v, o, lse, do, kp, vp, idx, blocks=blocks, **_ORC["flags"])
        _ORC["dq"][b, h, rows] = dq[0, 0, rows]
        with _ORC["locks"][head_no]:
            _ORC["dk"][b, h] += dk[0, 0]
            _ORC["dv"][b, h] += dv[0, 0]
    return len(blocks)


def host_cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OraclePool:
    """The oracle on ``cores`` worker processes over one workload's seeded inputs."""

    def __init__(self, cfg, host_inputs, flags: dict, cores: int | None = None):
        import multiprocessing as mp
        import numpy as np
        from multiprocessing import shared_memory

        self.cfg = cfg
        self.cores = cores or len(os.sched_getaffinity(0))
        B, H, N, D = cfg.B, cfg.H, cfg.N, cfg.D
        sizes = {"q": 4, "k": 4, "v": 4, "do": 4, "o": 8, "dq": 8, "dk": 8, "dv": 8}
        self.shm = {k: shared_memory.SharedMemory(create=True, size=B * H * N * D * w) for k, w in sizes.items()}
        self.shm["lse"] = shared_memory.SharedMemory(create=True, size=B * H * N * 8)
        for k in ("q", "k", "v", "do"):
            np.ndarray((B, H, N, D), dtype=np.float32, buffer=self.shm[k].buf)[...] = \
                host_inputs[k].float().numpy()
        self.dk = np.ndarray((B, H, N, D), dtype=np.float64, buffer=self.shm["dk"].buf)
        self.dv = np.ndarray((B, H, N, D), dtype=np.float64, buffer=self.shm["dv"].buf)
        ctx = mp.get_context("spawn")
        locks = [ctx.Lock() for _ in range(B * H)]
        self.pool = ctx.Pool(self.cores, initializer=_orc_attach,
                             initargs=({k: m.name for k, m in self.shm.items()}, (B, H, N, D), flags, cfg.levels,
                                       cfg.topk, locks))

    def step(self, heads=None, backward=None) -> float:
        """One oracle step over ``heads`` ((b, h) pairs; all by default); returns seconds."""
        import numpy as np
        cfg = self.cfg
        heads = heads or [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
        backward = cfg.backward if backward is None else backward
        n1 = cfg.N // 16
        chunks = max(1, min(n1, (2 * self.cores + len(heads) - 1) // len(heads)))
        t0 = time.perf_counter()
        for b, h in heads:
            self.dk[b, h] = 0.0
            self.dv[b, h] = 0.0
        per_head = self.pool.map(_orc_head, heads)
        tasks = []
        for no, (bh, (kp, vp, idx)) in enumerate(zip(heads, per_head)):
            for blocks in np.array_split(np.arange(n1), chunks):
                if blocks.size:
                    tasks.append((bh, blocks, kp, vp, idx, bh[0] * cfg.H + bh[1], backward))
        done = sum(self.pool.map(_orc_chunk, tasks, chunksize=1))
        assert done == n1 * len(heads)
        return time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()
        for m in self.shm.values():
            m.close()
            m.unlink()


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
    if args.grid_order:
        host = to_grid_order(host, cfg)
    pinned = {k: v.pin_memory() for k, v in host.items()}
    dev = {k: v.cuda(non_blocking=True) for k, v in pinned.items()}
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, dtype, grid_order=args.grid_order,
                           one_launch_select=args.one_launch_select, causal=args.causal, **enrichment(args))
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
    step_compulsory = compulsory_bytes(cfg, 2 if cfg.dtype == "bf16" else 4)
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
    step_kernels = ("attn_fwd_bf16", "attn_bwd_dq_bf16", "attn_bwd_dkdv_bf16", "pyramid_l12", "pyramid_select")
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
    in_mb = in_bytes / 1e6
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

    # forward only (pyramid, selection, forward: the inference path) and the standalone index
    # transpose, each timed eagerly on the launching stream after warm-up
    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b2.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b2) / reps

    fwd_ms = timed(lambda: api.llsa_forward_path(shape, dev["q"], dev["k"], dev["v"], buf), 20)
    forward_only = {"ms_per_step": round(fwd_ms, 4), "tokens_per_s": round(tokens_per_step / (fwd_ms / 1000.0), 1),
                    "calls": "llsa_build_pyramid + llsa_select + llsa_forward, eager on one stream"}
    tr_ms = timed(lambda: api.llsa_index_transpose(shape, buf.idx, buf.row_ptr, buf.col, buf.ws_transpose), 50)
    entries = sum(cfg.B * cfg.H * n * cfg.topk for n in cfg.level_sizes()[1:])
    tr_bytes = counts["transpose_hist"]["bytes"] + counts["transpose_scatter"]["bytes"] + \
        counts["transpose_bucket"]["bytes"] + counts.get("transpose_scan", {"bytes": 0})["bytes"]
    transpose = {"avg_us": round(1000 * tr_ms, 2), "entries": entries,
                 "entries_per_s": round(entries / (tr_ms / 1000.0), 1),
                 "gbs": round(tr_bytes / (tr_ms / 1000.0) / 1e9, 1),
                 "calls": "llsa_index_transpose (all levels, 4 launches), eager"}
    gather = measure_gather_peak(api, torch, stream, props.multi_processor_count)
    if roofline:
        c = counts[dominant]
        sec = kern[dominant]["avg_us"] * 1e-6
        roofline["l2_gather_peak_gbs"] = gather["gbs"]
        roofline["l2_frac"] = round(c["bytes"] / sec / 1e9 / gather["gbs"], 4)
        roofline["compulsory_frac"] = round(step_compulsory / (hbm_peak * 1e9) / (ms_per_step * 1e-3), 4)
        roofline["note"] = ("frac charges every gathered tile at HBM speed, but L2 serves most gathers, so "
                            "frac > 1 means the model overstates the HBM bytes; l2_frac is the same bytes "
                            "against the measured L2 -> SM tile-gather ceiling; compulsory_frac is the whole "
                            "step's unavoidable DRAM bytes at the HBM peak over the measured step time")
    for k, v in kernels_roof.items():
        if k.startswith("attn_"):
            c = counts[k]
            v["l2_frac"] = round(c["bytes"] / (kern[k]["avg_us"] * 1e-6) / 1e9 / gather["gbs"], 4)

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
        pool = OraclePool(cfg, host, enrichment(args))
        try:
            pool.step(heads=[(0, 0)])          # workers import the oracle and page in
            secs = pool.step(backward=True)    # the whole step the CUDA arm times
        finally:
            pool.close()
        cpu = {"value": round(tokens_per_step / secs, 2), "unit": UNIT, "cores": pool.cores, "kind": "oracle",
               "cpu_model": host_cpu_model(), "seconds": round(secs, 3),
               "sample": (f"the whole step of the workload (all {cfg.B * cfg.H} heads: pyramid, selection, "
                          f"index transpose, forward and backward), numpy fp64 oracle on {pool.cores} worker "
                          "processes (one thread each) over (head, query-block chunk)")}

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
                   "mask": "causal (LLSA_FLAG_CAUSAL)" if args.causal else "none (non-causal)",
                   "token_order": ("row-major grid, read and written through the quadtree order in the kernels "
                                   "(LLSA_FLAG_GRID_ORDER)" if args.grid_order else "quadtree (Z) order"),
                   "launch": ("K steps as one CUDA graph (llsa_plan_create repeat=K), kernels chained by "
                              "programmatic dependent launch; transpose on a second stream"
                              + ("; pyramid and selection as one cooperative launch (LLSA_FLAG_ONE_LAUNCH_SELECT)"
                                 if args.one_launch_select else "")),
                   "kernel_times_from": ("a second plan of the same K steps with trace events around every "
                                         f"kernel, launched after the timed one: {traced_ms_per_step:.4f} ms per step"),
                   "parallelism": f"dp{world}: independent replicas, no collective",
                   "l2": (f"inputs larger than L2: q, k, v, dO are {in_mb:.0f} MB per replica vs 126 MB L2; "
                          "no flush")},
        "roofline": roofline,
        "step_roofline": {"modelled_bytes": step_bytes, "flops": step_flops, "roofline_ms": round(step_roof_ms, 4),
                          "frac": round(step_roof_ms / ms_per_step, 4)},
        "compulsory": {"bytes": step_compulsory,
                       "floor_ms": round(1000 * step_compulsory / (hbm_peak * 1e9), 4),
                       "frac": round(1000 * step_compulsory / (hbm_peak * 1e9) / ms_per_step, 4),
                       "what": ("q, k, v, dO read once; o, dq, dk, dv, LSE, pyramids, selection and CSR "
                                "written once, at the measured HBM peak")},
        "l2_gather_peak": gather,
        "forward_only": forward_only,
        "index_transpose": transpose,
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
    """The CPU oracle as the reference arm, on every host core: rank 0 only.  Each step is the
    oracle's whole step over a sample of the workload's heads (all of them when that fits in
    about two and a half minutes for warm-up plus steps); the value is the sample's tokens
    (its share of B*N) per second of the sample's measured time, with nothing extrapolated."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    if args.causal:
        print(json.dumps({"impl": "reference", "unavailable": "the timed oracle arm covers the non-causal step only"}))
        return
    from synthetic import WORKLOADS, make_config_inputs

    wall0 = time.perf_counter()
    cfg = WORKLOADS[args.workload]
    host = make_config_inputs(cfg, with_do=True)
    pool = OraclePool(cfg, host, enrichment(args), cores=args.ref_cores)
    heads_all = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
    try:
        t_head = pool.step(heads=heads_all[:1], backward=True)
        per_step = len(heads_all)
        while per_step > 1 and (args.steps + args.warmup) * t_head * per_step > 150.0:
            per_step -= 1
        secs = []
        for i in range(args.warmup + args.steps):
            heads = [heads_all[(i * per_step + j) % len(heads_all)] for j in range(per_step)]
            t = pool.step(heads=heads, backward=True)
            if i >= args.warmup:
                secs.append(t)
    finally:
        pool.close()
    total_s = sum(secs)
    tokens_per_step = cfg.B * cfg.N * per_step / len(heads_all)
    value = tokens_per_step * args.steps / total_s
    ms_per_step = 1000.0 * total_s / args.steps
    sample = (f"numpy fp64 oracle on {pool.cores} worker processes ({host_cpu_model()}), per step the whole "
              f"step (pyramid, selection, index transpose, forward, backward) of {per_step} of the "
              f"{len(heads_all)} heads; value = those heads' share of the step's tokens per measured second")
    result = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": {"workload": f"{cfg.name}: {cfg.describe()}", "B": cfg.B, "H": cfg.H, "N": cfg.N, "D": cfg.D,
                   "block": cfg.block, "levels": cfg.levels, "topk": cfg.topk,
                   "kv_len": 16 * cfg.topk + (cfg.topk if args.level1 else 0) + coarse_entries(cfg, args.all_top),
                   "enrichment": enrichment_text(args),
                   "mask": "causal (LLSA_FLAG_CAUSAL)" if args.causal else "none (non-causal)", "heads_per_step": per_step,
                   "tokens_per_step": tokens_per_step},
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": pool.cores, "kind": "oracle",
                         "cpu_model": host_cpu_model(), "sample": sample},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    # the timed steps are whole oracle steps that ran inside this process: steps x ms_per_step is
    # measured time, not an extrapolation, and fits in the run's own wall clock
    wall = time.perf_counter() - wall0
    timed = args.steps * ms_per_step / 1000.0
    result["consistency"] = {"timed_seconds": round(timed, 3), "wall_seconds": round(wall, 3), "extrapolated": False,
                             "fits_in_driver_run": timed <= wall}
    print(json.dumps(result), flush=True)


def run_profile(args):
    """Only the timed step, for profilers: W warm-up steps then K steps, one line of output."""
    import torch

    from log_linear_hierarchical_b200 import api
    from synthetic import WORKLOADS, make_config_inputs

    cfg = WORKLOADS[args.workload]
    dtype = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    host = make_config_inputs(cfg, with_do=True)
    if args.grid_order:
        host = to_grid_order(host, cfg)
    dev = {k: v.cuda() for k, v in host.items()}
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, dtype, grid_order=args.grid_order,
                           one_launch_select=args.one_launch_select, causal=args.causal, **enrichment(args))
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
    ap.add_argument("--probe", action="store_true", help="run only the L2 gather-ceiling sweep (for ncu)")
    ap.add_argument("--log-bias", action="store_true",
                    help="the log-count enrichment variant (ln 16^l on level-l coarse scores)")
    ap.add_argument("--all-top", action="store_true",
                    help="the all-coarsest enrichment variant (every level-L token in every list)")
    ap.add_argument("--level1", action="store_true",
                    help="the level-1 enrichment variant (each selected block's mean token in the list)")
    ap.add_argument("--grid-order", action="store_true",
                    help="inputs and outputs in row-major grid order (LLSA_FLAG_GRID_ORDER)")
    ap.add_argument("--causal", action="store_true",
                    help="causal attention (LLSA_FLAG_CAUSAL; bf16, default enrichment)")
    ap.add_argument("--one-launch-select", action="store_true",
                    help="pyramid and selection as one cooperative launch (LLSA_FLAG_ONE_LAUNCH_SELECT)")
    ap.add_argument("--ref-cores", type=int, default=None,
                    help="worker processes of the reference arm's oracle (default: every host core)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.probe:
        run_probe(args)
    elif args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
