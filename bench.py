#!/usr/bin/env python
"""Packed-state decode benchmark on B200.

Workload: the 2,304-head GDN state pool (48 layers x 48 heads, d_k = d_v =
128) at 70 concurrent requests, nominal 6-bit plan over {4,6,8} with 32 FP16
pivot heads, synthetic seeded inputs.  A step is one decode step of every
(request, layer, head) state: reconstruct -> retention + delta update ->
readout -> refit r, c -> pack -> write back.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                    [--variant two_stream|fused] [--batch B] [--plan 6|4] [--no-sweep]
                    [--workload gdn|kda] [--scale-bits 32|16] [--shard replicas|layers]
                    [--prefill T [--prefill-kernel mma_sync|tcgen05]]

--prefill T times the chunked prefill of T-token prompt chunks into the
packed pool instead (tokens/s through the whole pool, tensor roofline).

The default single-GPU line also carries a sweep of workloads (batch
1/16/128/256 of the nominal-6 pool, the nominal-4 pool and bfloat16 scales at
batch 70, KDA rows at batch 128, the FP32-state step beside each) under
"sweep".

Prints one JSON line (rank 0).  N > 1: launched by torch.distributed.run, one
independent pool per GPU (no collective on the data path), barrier + max of
the per-rank device times; --shard layers splits one pool's layers instead.
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "packed-state decode head-steps/s and HBM GB/s (% of peak), 2304 heads, bs=70"
PREFILL_METRIC = "chunked prefill tokens/s into the packed state pool"
TF32_PER_BF16 = 1.1 / 2.25   # nominal dense TF32 / BF16 tensor throughput
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ["stepq_head.cu", "stepq_head.cuh", "stepq_head_tm.cu", "stepq_pipe.cuh", "stepq_dev.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="stepq", choices=["stepq", "reference"])
    ap.add_argument("--variant", default="fused", choices=["fused", "two_stream"])
    ap.add_argument("--batch", type=int, default=None, help="requests (default: 70 GDN pool, 128 KDA)")
    ap.add_argument("--plan", type=int, default=6, choices=[4, 6], help="nominal bits of the GDN pool plan")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "layers"],
                    help="replicas: one whole pool per rank (weak scaling); layers: one pool whose layers "
                         "are split over the ranks, each rank holding its layers' records (strong scaling)")
    ap.add_argument("--scale-bits", type=int, default=32, choices=[32, 16],
                    help="storage of the r and c scales in the plan (16: bfloat16)")
    ap.add_argument("--workload", default="gdn", choices=["gdn", "kda"],
                    help="gdn: 2,304-head pool; kda: 81,920 key rows (20 x 32 x 128)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the workload sweep that the default single-GPU line carries (batch 1/16/128/256, "
                         "nominal-4 plan, KDA rows at batch 128, 16-bit scales, the FP32-state kernel for each)")
    ap.add_argument("--prefill", type=int, default=0, metavar="T",
                    help="time chunked prefill of T-token prompt chunks into the packed pool (GDN) instead of "
                         "the decode step; batch defaults to 1")
    ap.add_argument("--prefill-kernel", default="tcgen05", choices=["mma_sync", "tcgen05"],
                    help="prefill kernel for per-head plans: the state in tensor memory with its products on "
                         "tcgen05 (default) or mma.sync tiles")
    ap.add_argument("--step-kernel", default="registers", choices=["registers", "tmem"],
                    help="fused step kernel for the per-head pool: state in registers (default) or in tensor memory")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle leg")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_init():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(x: float, ws: int, op):
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    return _reduce(x, ws, dist.ReduceOp.MAX)


def sum_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    return _reduce(x, ws, dist.ReduceOp.SUM)


def layer_range(L: int, ws: int, rank: int):
    """Layers [lb, le) of `rank` when a pool's L layers are split over ws ranks:
    contiguous ranges whose sizes differ by at most one, covering [0, L)."""
    if ws > L:
        raise ValueError(f"cannot split {L} layers over {ws} ranks")
    base, extra = divmod(L, ws)
    lb = rank * base + min(rank, extra)
    return lb, lb + base + (1 if rank < extra else 0)


def replica_throughput(units_local: float, secs_local: float, ws: int):
    """Whole-job throughput of independent replicas: all ranks' units over the
    slowest rank's device time.  Returns (units/s, max seconds)."""
    secs = max_over_ranks(secs_local, ws)
    return sum_over_ranks(units_local, ws) / secs, secs


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_tflops():
    """Dense bf16 tensor throughput measured by a cuBLAS GEMM burst (TFLOP/s)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(p))["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback"


def kernel_hash():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "quantized_recurrent_state_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_counts(variant: str):
    """(DRAM bytes, warp-instructions) per full launch from the committed ncu
    summary, each None unless it was taken on the current kernel source."""
    f = os.path.join(ROOT, "profiles", f"{variant}_kernel_traffic.txt")
    try:
        kv = dict(line.split(":", 1) for line in open(f) if ":" in line and not line.startswith("#"))
    except OSError:
        return None, None
    if kv.get("kernel_hash", "").strip() != kernel_hash():
        return None, None

    def num(key):
        try:
            return float(kv[key])
        except (KeyError, ValueError):
            return None
    return num("dram_bytes_per_full_launch"), num("warp_instructions_per_full_launch")


# SM issue peak: 4 schedulers per SM, one warp-instruction each per clock
def issue_peak(n_sms: int, mhz: float) -> float:
    return 4.0 * n_sms * mhz * 1e6


# ---------------------------------------------------------------------------
# product path
# ---------------------------------------------------------------------------

def product_plan(stepq, synth, wl, device, scale_bits=32):
    """Calibrate on the GPU (FP32-state recurrence + omega / log-gate /
    distortion kernels) and build the plan with the library's planner."""
    import torch
    L, H, D = wl.n_layers, wl.n_heads, wl.d
    bits = list(wl.bits)
    # a uniform plan at the largest width only to host the calibration kernels' context
    units = L * H if wl.mode == 0 else L * H * D
    dummy = stepq.Plan.build(wl.mode, L, H, D, bits, float(max(bits)), 0, wl.horizon, np.zeros(units),
                             np.tile(np.linspace(1.0, 0.25, len(bits)), (units, 1)), np.ones(L * H * D, np.float32))
    n = wl.calib_req
    ctx = stepq.Context(dummy, n)
    alpha = synth.gates(wl, wl.calib_seed)
    om = torch.zeros((L, H, D), dtype=torch.float64, device=device)
    ls = torch.zeros_like(om)
    S = torch.cat([synth.initial_states_torch(wl, wl.calib_seed, n, l, device) for l in range(L)], dim=1)
    slots = torch.arange(n, dtype=torch.int32, device=device)
    steps = [synth.step_inputs_torch(wl, wl.calib_seed, n, t, alpha, device) for t in range(wl.calib_steps)]
    for st in steps:
        ctx.calib_accumulate(n, 0, L, st["q"], st["k"], st["alpha"], st["beta"], om, ls)
    ctx.sync()
    omega = om.cpu().numpy() / (wl.calib_steps * n)
    lmean = ls.cpu().numpy() / (wl.calib_steps * n)
    wbar = np.maximum(omega / omega.mean(axis=2, keepdims=True), 1e-12).astype(np.float32)
    wbar_d = torch.from_numpy(wbar).to(device)
    dist = torch.zeros((L, H, D, len(bits)), dtype=torch.float64, device=device)
    o = torch.zeros((n, L, H, D), dtype=torch.float32, device=device)
    n_snap = 0
    for t, st in enumerate(steps):
        ctx.fp32_decode_step(S, slots, n, 0, L, st["q"], st["k"], st["v"], st["alpha"], st["beta"], o)
        if (t + 1) % 8 == 0:
            ctx.calib_distortion(n, 0, L, S, wbar_d, bits, dist)
            n_snap += 1
    ctx.sync()
    d = dist.cpu().numpy() / (n_snap * n)
    ctx.close()
    import tempfile
    fd, path = tempfile.mkstemp(suffix=".plan")
    os.close(fd)
    if wl.mode == 0:
        lgate, dist = lmean.mean(axis=2).reshape(-1), d.sum(axis=2).reshape(-1, len(bits))
    else:
        lgate, dist = lmean.reshape(-1), d.reshape(-1, len(bits))
    plan = stepq.Plan.build(wl.mode, L, H, D, bits, wl.nominal_bits, wl.n_pivots, wl.horizon,
                            lgate, dist, wbar.reshape(-1), path=path, scale_bits=scale_bits)
    data = open(path, "rb").read()
    os.unlink(path)
    return plan, data


def gate_bytes(plan):
    """alpha + beta bytes of one head-step: scalar alpha (GDN) or one per key row (KDA)."""
    return (4 if plan.mode == 0 else 4 * plan.d) + 4


def step_bytes(plan, n_req):
    """Algorithmic bytes of one single-pass step: every record read and
    written once, q, k, v read, o written, alpha and beta read."""
    L, H, D = plan.n_layers, plan.n_heads, plan.d
    rec = 0
    for l in range(L):
        for h in range(H):
            rec += plan.record(l, h)[1]
    per_slot = 2 * rec + L * H * (3 * 4 * D + gate_bytes(plan) + 4 * D)
    return per_slot * n_req


def kernel_bytes(plan, n_req, kind):
    """Algorithmic bytes per launch of the per-kernel roofline: decode reads
    records, q, k, v, alpha, beta and writes o, w; fit-pack reads records, k,
    w, alpha, beta and writes records."""
    L, H, D = plan.n_layers, plan.n_heads, plan.d
    rec = sum(plan.record(l, h)[1] for l in range(L) for h in range(H))
    if kind == "fused":
        return step_bytes(plan, n_req)
    if kind == "decode":
        return n_req * (rec + L * H * (3 * 4 * D + gate_bytes(plan) + 2 * 4 * D))
    return n_req * (2 * rec + L * H * (2 * 4 * D + gate_bytes(plan)))


def run_step(ctx, variant, pool, slots, n, L, inp, o, ws):
    if variant == "fused":
        ctx.decode_step_fused(pool, slots, n, 0, L, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o)
    else:
        ctx.decode_step(pool, slots, n, 0, L, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, ws)


def time_steps(torch, ctx, variant, pool, slots, n, L, sets, o, ws, warmup, steps, ws_ranks, clocks=None):
    """Device time of `steps` steps (CUDA events on the main stream, which
    waits for the side stream at the end); returns (seconds, kernel stats)."""
    main, side = ctx.main, ctx.side
    for i in range(warmup):
        run_step(ctx, variant, pool, slots, n, L, sets[i % len(sets)], o, ws)
    ctx.sync()
    ctx.kernel_stats()
    torch.cuda.synchronize()
    barrier(ws_ranks)
    torch.cuda.synchronize()
    ctx.set_timing(True)
    launches0 = ctx.launches
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    join = torch.cuda.Event()
    if clocks:
        clocks.__enter__()
    e0.record(main)
    for i in range(steps):
        run_step(ctx, variant, pool, slots, n, L, sets[i % len(sets)], o, ws)
    join.record(side)
    main.wait_event(join)
    e1.record(main)
    torch.cuda.synchronize()
    if clocks:
        clocks.__exit__(None, None, None)
    ctx.sync()
    barrier(ws_ranks)
    torch.cuda.synchronize()
    ctx.set_timing(False)
    launches = ctx.launches - launches0
    stats = ctx.kernel_stats()
    return e0.elapsed_time(e1) / 1e3, stats, launches


def workload_of(args, synth):
    if args.workload == "kda":
        wl = synth.workloads()["kda_rows"]
    else:
        wl = synth.workloads()["qwen_pool6" if args.plan == 6 else "qwen_pool4"]
    if args.batch is None:
        args.batch = 1 if args.prefill else 128 if args.workload == "kda" else 70
    return wl


def workload_config(wl, n, ws):
    """The `config` keys both arms print for the same workload."""
    L, H, D = wl.n_layers, wl.n_heads, wl.d
    if wl.mode == 0:
        name = (f"GDN state pool, {L} layers x {H} heads = {L * H} heads, d_k=d_v={D}, batch {n}, "
                f"nominal {wl.nominal_bits:g}-bit plan over {sorted(wl.bits)}, {wl.n_pivots} FP16 pivot heads")
    else:
        name = (f"KDA per-key-row units, {L} layers x {H} heads x {D} rows = {L * H * D} rows, d_v={D}, "
                f"batch {n}, Lagrangian nominal {wl.nominal_bits:g}-bit plan over {sorted(wl.bits)}, "
                f"{wl.n_pivots} FP16 pivot rows, per-row gates")
    return {"workload": name, "batch": n, "heads": L * H, "d": D,
            "l2": "inputs larger than L2 (pool and q/k/v far above 126 MB)",
            "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"}


def variant_is_full_launch(args) -> bool:
    """The committed instruction count is for the default full launch (fused,
    GDN pool, batch 70, nominal 6, fp32 scales)."""
    return (args.variant == "fused" and args.workload == "gdn" and args.batch == 70 and args.plan == 6
            and args.scale_bits == 32 and args.shard == "replicas")


def measure_packed(torch, stepq, synth, wl, plan, n, device, steps=12, warmup=3, step_kernel=0):
    """Fused packed step of a whole pool at batch n: CUDA-event time of `steps`
    steps on the context's main stream."""
    L, H, D = wl.n_layers, wl.n_heads, wl.d
    ctx = stepq.Context(plan, n)
    ctx.set_step_kernel(step_kernel)
    pool = torch.zeros(n * plan.slot_bytes, dtype=torch.uint8, device=device)
    slots = torch.arange(n, dtype=torch.int32, device=device)
    for l in range(L):
        ctx.requant_pack(pool, slots, n, l, l + 1, synth.initial_states_torch(wl, wl.seed, n, l, device))
    alpha = synth.gates(wl, wl.seed)
    sets = [synth.step_inputs_torch(wl, wl.seed, n, t, alpha, device) for t in range(2)]
    o = torch.zeros((n, L, H, D), dtype=torch.float32, device=device)
    ctx.sync()
    secs, stats, _ = time_steps(torch, ctx, "fused", pool, slots, n, L, sets, o, None, warmup, steps, 1)
    k_ms, k_n = stats["fused"]
    ctx.close()
    del pool, sets, o
    torch.cuda.empty_cache()
    return secs / steps, (k_ms / k_n / 1e3) if k_n else None


def measure_fp32(torch, stepq, synth, wl, plan, n, device, steps=6, warmup=2):
    """The FP32-state step on the same pool shape at batch n (seconds per step)."""
    L, H, D = wl.n_layers, wl.n_heads, wl.d
    ctx = stepq.Context(plan, n)
    S32 = torch.empty((n, L, H, D, D), dtype=torch.float32, device=device)
    for l in range(L):
        S32[:, l:l + 1] = synth.initial_states_torch(wl, wl.seed, n, l, device)
    slots = torch.arange(n, dtype=torch.int32, device=device)
    alpha = synth.gates(wl, wl.seed)
    sets = [synth.step_inputs_torch(wl, wl.seed, n, t, alpha, device) for t in range(2)]
    o = torch.zeros((n, L, H, D), dtype=torch.float32, device=device)
    for i in range(warmup):
        x = sets[i % 2]
        ctx.fp32_decode_step(S32, slots, n, 0, L, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(ctx.main)
    for i in range(steps):
        x = sets[i % 2]
        ctx.fp32_decode_step(S32, slots, n, 0, L, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o)
    e1.record(ctx.main)
    torch.cuda.synchronize()
    ctx.close()
    del S32, sets, o
    torch.cuda.empty_cache()
    return e0.elapsed_time(e1) / 1e3 / steps


def workload_sweep(torch, stepq, synth, device, plan6, peak, step_kernel=0):
    """The configurations the single-GPU line reports beside the headline: the
    nominal-6 pool at batch 1/16/128/256, the nominal-4 pool over {2,4,6,8} and
    16-bit scales at batch 70, KDA per-key-row units at batch 128, each with the
    FP32-state step on the same pool shape.  Per entry: head-steps/s, tokens/s
    (state updates of a request across the whole pool), algorithmic GB/s of the
    single-pass step and its fraction of the measured peak."""
    out = []

    def entry(name, wl, plan, n, fp32=True):
        t, t_k = measure_packed(torch, stepq, synth, wl, plan, n, device, step_kernel=step_kernel)
        L, H, D = wl.n_layers, wl.n_heads, wl.d
        b = step_bytes(plan, n)
        e = {"config": name, "batch": n, "ms_per_step": t * 1e3, "head_steps_per_s": n * L * H / t,
             "tokens_per_s": n / t, "gbs": b / t / 1e9, "frac": b / t / 1e9 / peak,
             "kernel_ms": t_k * 1e3 if t_k else None, "bits_per_value": plan.info.bits_per_value,
             "bits_per_value_s16": plan.info.bits_per_value_s16}
        if n == 1:
            e["l2"] = "the whole pool fits in the 126 MB L2 and stays there between steps"
        if fp32:
            t32 = measure_fp32(torch, stepq, synth, wl, plan, n, device)
            b32 = n * L * H * (2 * 4 * D * D + 3 * 4 * D + gate_bytes(plan) + 4 * D)
            e["fp32_state"] = {"ms_per_step": t32 * 1e3, "head_steps_per_s": n * L * H / t32,
                               "gbs": b32 / t32 / 1e9, "frac": b32 / t32 / 1e9 / peak,
                               "packed_speedup": t32 / t}
        out.append(e)

    wl6 = synth.workloads()["qwen_pool6"]
    for n in (1, 16, 128, 256):
        entry("GDN pool, nominal 6 over {4,6,8}, 32 pivots", wl6, plan6, n)
    wl4 = synth.workloads()["qwen_pool4"]
    plan4, _ = product_plan(stepq, synth, wl4, device)
    entry("GDN pool, nominal 4 over {2,4,6,8}, 32 pivots", wl4, plan4, 70, fp32=False)
    plan16, _ = product_plan(stepq, synth, wl6, device, scale_bits=16)
    entry("GDN pool, nominal 6, bfloat16 r and c", wl6, plan16, 70, fp32=False)
    wlk = synth.workloads()["kda_rows"]
    plank, _ = product_plan(stepq, synth, wlk, device)
    entry("KDA per-key-row units, 81,920 rows, nominal 6 over {4,6,8}, 512 pivot rows", wlk, plank, 128)
    return out


def run_product(args):
    import torch
    from quantized_recurrent_state_b200 import build as qbuild
    ws, rank, local = dist_init()
    if rank == 0:
        qbuild.build()
    barrier(ws)
    from quantized_recurrent_state_b200 import stepq, synth
    device = torch.device("cuda", local)
    wl = workload_of(args, synth)
    n = args.batch
    plan, plan_bytes = product_plan(stepq, synth, wl, device, args.scale_bits)
    H, D = wl.n_heads, wl.d
    lb, le = (0, wl.n_layers) if args.shard == "replicas" else layer_range(wl.n_layers, ws, rank)
    if args.shard == "layers":
        plan = plan.slice(lb, le)   # this rank holds the records of its own layers only
    L = le - lb
    step_kernel = stepq.STEP_TMEM if args.step_kernel == "tmem" else stepq.STEP_REGISTERS
    ctx = stepq.Context(plan, n)
    ctx.set_step_kernel(step_kernel)
    pool = torch.zeros(n * plan.slot_bytes, dtype=torch.uint8, device=device)
    slots = torch.arange(n, dtype=torch.int32, device=device)
    for l in range(L):
        ctx.requant_pack(pool, slots, n, l, l + 1, synth.initial_states_torch(wl, wl.seed, n, lb + l, device))
    ctx.sync()
    alpha = synth.gates(wl, wl.seed)
    sets = [{k: v[:, lb:le].contiguous() for k, v in synth.step_inputs_torch(wl, wl.seed, n, t, alpha, device).items()}
            for t in range(4)]
    o = torch.zeros((n, L, H, D), dtype=torch.float32, device=device)
    wsp = torch.empty(ctx.workspace_bytes(n, L) // 4, dtype=torch.float32, device=device)
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    secs, stats, launches = time_steps(torch, ctx, args.variant, pool, slots, n, L, sets, o, wsp,
                                       args.warmup, args.steps, ws, clocks)
    head_steps = n * L * H * args.steps
    value, secs = replica_throughput(head_steps, secs, ws)
    sb = step_bytes(plan, n)
    gbs = sb * args.steps / secs / 1e9
    peak, peak_kind = measured_peaks()

    # dominant kernel of the variant: its own algorithmic bytes over its mean launch time
    kind = "fused" if args.variant == "fused" else max(("decode", "fitpack"), key=lambda k: stats[k][0])
    k_ms, k_n = stats[kind]
    # algorithmic bytes of one launch: the kernel's bytes per step over its launches per step
    k_bytes = kernel_bytes(plan, n, kind) / (k_n / args.steps) if k_n else None
    achieved = k_bytes / (k_ms / k_n / 1e3) / 1e9 if k_n else None
    traffic, winst = profiled_counts(args.variant) if variant_is_full_launch(args) else (None, None)

    extra = {}
    # FP32-state reference kernel: same workload, fp32 state pool
    if rank == 0:
        S32 = torch.empty((n, L, H, D, D), dtype=torch.float32, device=device)
        for l in range(L):
            S32[:, l:l + 1] = synth.initial_states_torch(wl, wl.seed, n, lb + l, device)
        for i in range(2):
            ctx.fp32_decode_step(S32, slots, n, 0, L, sets[i]["q"], sets[i]["k"], sets[i]["v"], sets[i]["alpha"],
                                 sets[i]["beta"], o)
        torch.cuda.synchronize()
        reps = 4
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(ctx.main)
        for i in range(reps):
            ctx.fp32_decode_step(S32, slots, n, 0, L, sets[i % 4]["q"], sets[i % 4]["k"], sets[i % 4]["v"],
                                 sets[i % 4]["alpha"], sets[i % 4]["beta"], o)
        e1.record(ctx.main)
        torch.cuda.synchronize()
        t32 = e0.elapsed_time(e1) / 1e3 / reps
        b32 = n * L * H * (2 * 4 * D * D + 3 * 4 * D + gate_bytes(plan) + 4 * D)
        extra["fp32_state_kernel"] = {"head_steps_per_s": n * L * H / t32, "ms_per_step": t32 * 1e3,
                                      "gbs": b32 / t32 / 1e9, "frac": b32 / t32 / 1e9 / peak}
        del S32
        torch.cuda.empty_cache()
        # in-run stream-copy peak
        nb = 4 << 30
        a = torch.empty(nb, dtype=torch.uint8, device=device)
        b = torch.empty_like(a)
        stream = torch.cuda.current_stream()
        stepq.copy_probe(b, a, nb, stream)
        best = 0.0
        for _ in range(10):
            c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            c0.record(stream)
            stepq.copy_probe(b, a, nb, stream)
            c1.record(stream)
            torch.cuda.synchronize()
            best = max(best, 2 * nb / (c0.elapsed_time(c1) / 1e3) / 1e9)
        extra["copy_probe_gbs"] = best
        extra["kernel_frac_of_copy_probe"] = achieved / best if achieved else None
        del a, b
        torch.cuda.empty_cache()

    # end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        # Every step: its q, k, v, alpha, beta copied from pinned host memory, the step, and
        # o copied back to pinned host memory.  Two input/output buffer sets let step i's
        # upload (split over two copy streams) and step i-1's download overlap step i-1's kernels.
        NB = 2
        host = {k: v.cpu().pin_memory() for k, v in sets[0].items()}
        dev_in = [{k: torch.empty_like(v) for k, v in sets[0].items()} for _ in range(NB)]
        o_dev = [torch.empty_like(o) for _ in range(NB)]
        o_host = [torch.empty(o.shape, dtype=torch.float32).pin_memory() for _ in range(NB)]
        ups, down = (torch.cuda.Stream(), torch.cuda.Stream()), torch.cuda.Stream()
        split = (("q", "k"), ("v", "alpha", "beta"))
        ev_in = [[torch.cuda.Event() for _ in ups] for _ in range(NB)]
        ev_done = [torch.cuda.Event() for _ in range(NB)]
        ev_out = [torch.cuda.Event() for _ in range(NB)]
        h2d = sum(v.numel() * 4 for v in host.values())
        d2h = o_host[0].numel() * 4
        k_e2e = args.steps
        torch.cuda.synchronize()
        barrier(ws)
        t0 = time.perf_counter()
        for i in range(k_e2e):
            bi = i % NB
            for si, up in enumerate(ups):
                with torch.cuda.stream(up):
                    if i >= NB:
                        up.wait_event(ev_done[bi])  # step i-NB no longer reads these inputs
                    for kk in split[si]:
                        dev_in[bi][kk].copy_(host[kk], non_blocking=True)
                    ev_in[bi][si].record(up)
            with torch.cuda.stream(ctx.main):
                for ev in ev_in[bi]:
                    ctx.main.wait_event(ev)
                if i >= NB:
                    ctx.main.wait_event(ev_out[bi])  # o of step i-NB is on the host
                run_step(ctx, args.variant, pool, slots, n, L, dev_in[bi], o_dev[bi], wsp)
                ctx.main.wait_stream(ctx.side)
                ev_done[bi].record(ctx.main)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[bi])
                o_host[bi].copy_(o_dev[bi], non_blocking=True)
                ev_out[bi].record(down)
        ctx.sync()
        torch.cuda.synchronize()
        t_e2e = max_over_ranks(time.perf_counter() - t0, ws)
        e2e = {"value": sum_over_ranks(n * L * H * k_e2e, ws) / t_e2e, "unit": "head-steps/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k_e2e,
               "overlap": "uploads (two streams) and downloads (one) double-buffered, overlapping the steps"}

    sweep = None
    if (rank == 0 and ws == 1 and not args.no_sweep and args.workload == "gdn" and args.plan == 6
            and args.scale_bits == 32 and args.variant == "fused" and args.batch == 70):
        sweep = workload_sweep(torch, stepq, synth, device, plan, peak, step_kernel)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        cpu = cpu_baseline(plan_bytes, wl, budget_s=12.0)

    if rank == 0:
        csum = clocks.summary()
        issue_view = None
        if winst and k_n and variant_is_full_launch(args):
            n_sms = torch.cuda.get_device_properties(device).multi_processor_count
            ach = winst / (k_ms / k_n * 1e-3)
            pk = issue_peak(n_sms, csum["sm_mhz"] or csum["sm_max_mhz"])
            issue_view = {"achieved": ach, "peak": pk, "unit": "warp-inst/s", "frac": ach / pk,
                          "instructions_per_launch": winst,
                          "note": "what binds the kernel: instruction issue (4 per SM per clock at the sampled clock)"}
        out = {
            "metric": METRIC,
            "value": value,
            "unit": "head-steps/s",
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True,
            "scaling": "weak" if args.shard == "replicas" else "strong",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic",
            "config": {
                **workload_config(wl, n, ws),
                **({"parallelism": f"layer shards x{ws} (rank 0: layers {lb}-{le - 1})"} if args.shard == "layers" else {}),
                "variant": args.variant,
                "step_kernel": args.step_kernel if (args.variant == "fused" and wl.mode == 0) else "registers",
                "bits_per_value": plan.info.bits_per_value, "bits_per_value_s16": plan.info.bits_per_value_s16,
                "scale_bits": plan.info.scale_bits, "pool_bytes": n * plan.slot_bytes,
            },
            "hbm_gbs": gbs,
            "hbm_frac": gbs / peak,
            "tokens_per_s": sum_over_ranks(n * args.steps, ws) / secs,
            "roofline": {"bound": "hbm", "kernel": kind, "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak if achieved else None, "traffic": traffic,
                         "algorithmic_bytes_per_launch": k_bytes, "launch_ms": k_ms / k_n if k_n else None,
                         "peak_source": peak_kind,
                         "issue": issue_view},
            "kernel_ms": {k: v[0] for k, v in stats.items() if v[1]},
            "kernel_launches": {k: v[1] for k, v in stats.items() if v[1]},
            "gpu_launches": launches,
            "clocks": {"sm_mhz": csum["sm_mhz"], "sm_max_mhz": csum["sm_max_mhz"], "reasons": csum["reasons"]},
            "e2e": e2e,
            "cpu_baseline": cpu,
            **extra,
        }
        if sweep:
            out["sweep"] = sweep
        print(json.dumps(out), flush=True)
    ctx.close()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# chunked prefill
# ---------------------------------------------------------------------------

PREFILL_CHUNK = 64   # tokens per chunk of the prefill kernel
PREFILL_CPU_TOKENS = 256   # tokens per head of the oracle's timed sample


def prefill_flops(T: int, D: int, C: int = PREFILL_CHUNK) -> int:
    """Algorithmic FLOPs of one head's T-token prefill in the chunk form: per
    chunk of c tokens the six dense products (K K^T, Q K^T, A U: 2 c^2 D each;
    K S_0, Q S_0, K^T U: 2 c D^2 each) and the triangular solve (c (c-1) D)."""
    tot = 0
    for c0 in range(0, T, C):
        c = min(C, T - c0)
        tot += 6 * c * c * D + 6 * c * D * D + c * (c - 1) * D
    return tot


def prefill_bytes(T: int, D: int, rows: bool = False) -> int:
    """Algorithmic HBM bytes of one head in a prefill kernel launch: q, k, v
    read and o written per token, alpha (one per head, or one per key row)
    and beta read, the fp32 state read and written once."""
    return T * (4 * 4 * D + (4 * D if rows else 4) + 4) + 2 * 4 * D * D


def prefill_config(wl, n, T, ws):
    L, H, D = wl.n_layers, wl.n_heads, wl.d
    pool = (f"the GDN state pool, {L} layers x {H} heads = {L * H} heads, d_k=d_v={D}, batch {n}, nominal "
            f"{wl.nominal_bits:g}-bit plan over {sorted(wl.bits)}, {wl.n_pivots} FP16 pivot heads" if wl.mode == 0 else
            f"the KDA per-key-row pool, {L} layers x {H} heads x {D} rows, d_v={D}, batch {n}, Lagrangian nominal "
            f"{wl.nominal_bits:g}-bit plan over {sorted(wl.bits)}, {wl.n_pivots} FP16 pivot rows, per-row gates")
    return {"workload": (f"chunked prefill of {T}-token prompt chunks into {pool}; each step continues from the "
                         f"packed states the previous one wrote"),
            "batch": n, "prompt_chunk_tokens": T, "kernel_chunk_tokens": PREFILL_CHUNK, "heads": L * H, "d": D,
            "l2": "inputs larger than L2 (one step's q, k, v far above 126 MB)",
            "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"}


def run_prefill(args):
    """One step = the packed prefill of a T-token chunk for every (request,
    layer, head): unpack the records, the chunked gated delta rule on the
    tensor cores, requantize and pack (three launches)."""
    import torch
    from quantized_recurrent_state_b200 import build as qbuild
    ws, rank, local = dist_init()
    if rank == 0:
        qbuild.build()
    barrier(ws)
    from quantized_recurrent_state_b200 import stepq, synth
    device = torch.device("cuda", local)
    wl = workload_of(args, synth)
    n, T = args.batch, args.prefill
    plan, plan_bytes = product_plan(stepq, synth, wl, device, args.scale_bits)
    H, D = wl.n_heads, wl.d
    lb, le = (0, wl.n_layers) if args.shard == "replicas" else layer_range(wl.n_layers, ws, rank)
    if args.shard == "layers":
        plan = plan.slice(lb, le)   # this rank holds the records of its own layers only
    L = le - lb
    ctx = stepq.Context(plan, n)
    ctx.set_prefill_kernel(stepq.PREFILL_TCGEN05 if args.prefill_kernel == "tcgen05" else stepq.PREFILL_MMA_SYNC)
    pool = torch.zeros(n * plan.slot_bytes, dtype=torch.uint8, device=device)
    slots = torch.arange(n, dtype=torch.int32, device=device)
    for l in range(L):
        ctx.requant_pack(pool, slots, n, l, l + 1, synth.initial_states_torch(wl, wl.seed, n, lb + l, device))
    alpha = synth.gates(wl, wl.seed)
    inp = synth.prompt_inputs_torch(wl, wl.seed, n, 0, T, alpha, device, lb, le)
    o = torch.zeros_like(inp["q"])
    wsp = torch.empty(ctx.prefill_workspace_bytes(n, L) // 4, dtype=torch.float32, device=device)
    torch.cuda.synchronize()

    def step():
        ctx.prefill(pool, slots, n, 0, L, T, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, wsp)

    for _ in range(args.warmup):
        step()
    ctx.sync()
    ctx.kernel_stats()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    ctx.set_timing(True)
    launches0 = ctx.launches
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.__enter__()
    e0.record(ctx.main)
    for _ in range(args.steps):
        step()
    e1.record(ctx.main)
    torch.cuda.synchronize()
    clocks.__exit__(None, None, None)
    ctx.sync()
    barrier(ws)
    torch.cuda.synchronize()
    ctx.set_timing(False)
    launches = ctx.launches - launches0
    stats = ctx.kernel_stats()
    # head-tokens summed over ranks, over the pool's heads: tokens through the whole pool
    # (replicas: every replica's pool; layer shards: the one pool they split)
    head_tokens, secs = replica_throughput(n * T * args.steps * L * H, e0.elapsed_time(e1) / 1e3, ws)
    value = head_tokens / (wl.n_layers * H)

    k_ms, k_n = stats["prefill"]
    launch_s = k_ms / k_n / 1e3
    flops = n * L * H * prefill_flops(T, D)
    bf16, peak_kind = measured_bf16_tflops()
    peak = bf16 * TF32_PER_BF16
    achieved = flops / launch_s / 1e12
    hbm_peak, hbm_kind = measured_peaks()
    k_bytes = n * L * H * prefill_bytes(T, D, wl.mode == 1)

    # the same tokens stepped one at a time by the fused decode step, for comparison
    compare = None
    if rank == 0:
        sets = [{k: v[:, lb:le].contiguous() for k, v in synth.step_inputs_torch(wl, wl.seed, n, t, alpha, device).items()}
                for t in range(4)]
        o2 = torch.zeros((n, L, H, D), dtype=torch.float32, device=device)
        w2 = torch.empty(ctx.workspace_bytes(n, L) // 4, dtype=torch.float32, device=device)
        sec_dec, _, _ = time_steps(torch, ctx, "fused", pool, slots, n, L, sets, o2, w2, 3, 32, 1)
        dec_tok = sec_dec / 32
        pre_tok = e0.elapsed_time(e1) / 1e3 / (args.steps * T)
        compare = {"fused_decode_ms_per_token": dec_tok * 1e3, "prefill_ms_per_token": pre_tok * 1e3,
                   "speedup": dec_tok / pre_tok,
                   "note": "per prompt token of the whole pool at this batch: the fused decode step run once "
                           "per token against the chunked prefill"}
        del sets, o2, w2

    e2e = None
    if not args.no_e2e:
        # every step: the chunk's q, k, v, alpha, beta from pinned host memory, the prefill, o back
        host = {k: v.cpu().pin_memory() for k, v in inp.items()}
        o_host = torch.empty(o.shape, dtype=torch.float32).pin_memory()
        h2d = sum(v.numel() * 4 for v in host.values())
        d2h = o_host.numel() * 4
        k_e2e = min(args.steps, 3)
        torch.cuda.synchronize()
        barrier(ws)
        t0 = time.perf_counter()
        for _ in range(k_e2e):
            with torch.cuda.stream(ctx.main):
                for kk in host:
                    inp[kk].copy_(host[kk], non_blocking=True)
                step()
                o_host.copy_(o, non_blocking=True)
        torch.cuda.synchronize()
        t_e2e = max_over_ranks(time.perf_counter() - t0, ws)
        e2e = {"value": sum_over_ranks(n * T * k_e2e * L * H, ws) / (wl.n_layers * H) / t_e2e, "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k_e2e,
               "overlap": "none: the copies and the launches of a step in order on one stream"}
        del host, o_host

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        cpu = cpu_prefill_baseline(plan_bytes, wl, budget_s=12.0)

    if rank == 0:
        csum = clocks.summary()
        out = {
            "metric": PREFILL_METRIC,
            "value": value,
            "unit": "tokens/s",
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True,
            "scaling": "weak" if args.shard == "replicas" else "strong",
            "vs_baseline": None,
            "dtype": "f32 (tensor-core products in TF32 with a TF32 remainder)",
            "data": "synthetic",
            "config": {**prefill_config(wl, n, T, ws), "scale_bits": plan.info.scale_bits,
                       "pool_bytes": n * plan.slot_bytes,
                       "prefill_kernel": args.prefill_kernel if wl.mode == 0 else "mma_sync",
                       **({"parallelism": f"layer shards x{ws} (rank 0: layers {lb}-{le - 1})"}
                          if args.shard == "layers" else {})},
            "head_tokens_per_s": head_tokens,
            "roofline": {"bound": "tensor", "kernel": "prefill", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                         "algorithmic_flops_per_launch": flops, "launch_ms": launch_s * 1e3,
                         "peak_source": f"{peak_kind} bf16 burst {bf16:g} TFLOP/s x nominal TF32/BF16 "
                                        f"{TF32_PER_BF16:.4f}",
                         "hbm": {"achieved": k_bytes / launch_s / 1e9, "peak": hbm_peak, "unit": "GB/s",
                                 "frac": k_bytes / launch_s / 1e9 / hbm_peak, "peak_source": hbm_kind,
                                 "algorithmic_bytes_per_launch": k_bytes},
                         "note": "each product runs as three TF32 MMAs (hi*hi + hi*lo + lo*hi), so the tensor "
                                 "pipe caps frac at 1/3"},
            "kernel_ms": {k: v[0] for k, v in stats.items() if v[1]},
            "kernel_launches": {k: v[1] for k, v in stats.items() if v[1]},
            "gpu_launches": launches,
            "clocks": {"sm_mhz": csum["sm_mhz"], "sm_max_mhz": csum["sm_max_mhz"], "reasons": csum["reasons"]},
            "vs_decode_loop": compare,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(out), flush=True)
    ctx.close()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# CPU oracle (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def _oracle_sample(payload):
    """One decode step of a set of (layer, head) states of request 0 with the
    oracle.  Packing S_0 and drawing inputs are not timed; returns the seconds
    spent stepping."""
    import numpy as np
    from oracle import model, plan_io
    from quantized_recurrent_state_b200 import synth
    plan_bytes, wname, heads, t = payload
    plan = plan_io.read_plan(plan_bytes)
    pv = model.PlanView(plan)
    wl = synth.workloads()[wname]
    alpha = synth.gates(wl, wl.seed)
    layers = sorted({l for l, _ in heads})
    inp = synth.step_inputs(wl, wl.seed, 1, t, alpha=alpha, layers=layers)
    slot = np.zeros(pv.slot_bytes, np.uint8)
    for li, l in enumerate(layers):
        S0 = synth.initial_states(wl, wl.seed, 1, layers=[l])
        for (l2, h) in heads:
            if l2 == l:
                pv.quantize_into(slot, l, h, S0[0, 0, h])
    t0 = time.perf_counter()
    for (l, h) in heads:
        li = layers.index(l)
        pv.step(slot, l, h, inp["q"][0, li, h], inp["k"][0, li, h], inp["v"][0, li, h],
                inp["alpha"][0, li, h], inp["beta"][0, li, h])
    return time.perf_counter() - t0


def _oracle_prefill_sample(payload):
    """The oracle's packed prefill of a T-token chunk for a set of (layer,
    head) states of request 0: reconstruct the record, the chunk form of the
    gated delta rule in fp64, requantize.  Packing S_0 and drawing inputs are
    not timed; returns the seconds spent."""
    import numpy as np
    from oracle import model, plan_io, prefill
    from quantized_recurrent_state_b200 import synth
    plan_bytes, wname, heads, T = payload
    chunked = prefill.chunked_rows if synth.workloads()[wname].mode == 1 else prefill.chunked
    pv = model.PlanView(plan_io.read_plan(plan_bytes))
    wl = synth.workloads()[wname]
    alpha = synth.gates(wl, wl.seed)
    layers = sorted({l for l, _ in heads})
    steps = [synth.step_inputs(wl, wl.seed, 1, t, alpha=alpha, layers=layers) for t in range(T)]
    seq = {k: np.stack([st[k][0] for st in steps]) for k in steps[0]}   # [T, nL, H(, D)]
    slot = np.zeros(pv.slot_bytes, np.uint8)
    for l in layers:
        S0 = synth.initial_states(wl, wl.seed, 1, layers=[l])
        for (l2, h) in heads:
            if l2 == l:
                pv.quantize_into(slot, l, h, S0[0, 0, h])
    t0 = time.perf_counter()
    for (l, h) in heads:
        li = layers.index(l)
        S = pv.reconstruct(slot, l, h).astype(np.float64)
        _, S_T = chunked(S, seq["q"][:, li, h], seq["k"][:, li, h], seq["v"][:, li, h],
                         seq["alpha"][:, li, h], seq["beta"][:, li, h])
        pv.quantize_into(slot, l, h, S_T)
    return time.perf_counter() - t0


def cpu_prefill_rate(plan_bytes, wl, n_heads, T, pool, cores):
    """Tokens/s (a token through all L*H heads) of the oracle's packed prefill
    over a sample of n_heads heads, split across the worker processes; the
    time is the slowest worker's."""
    heads = [(l, h) for l in range(wl.n_layers) for h in range(wl.n_heads)][:n_heads]
    chunks = [heads[i::cores] for i in range(cores)]
    secs = max(pool.map(_oracle_prefill_sample, [(plan_bytes, wl.name, c, T) for c in chunks if c]))
    return len(heads) * T / (wl.n_layers * wl.n_heads) / secs, len(heads), secs


def cpu_prefill_baseline(plan_bytes, wl, budget_s=12.0):
    cores = _n_cores()
    T = PREFILL_CPU_TOKENS
    per_head = _oracle_prefill_sample((plan_bytes, wl.name, [(0, 0)], T))
    nh = int(min(wl.n_layers * wl.n_heads, max(cores, budget_s / max(per_head, 1e-4))))
    with oracle_pool(cores) as pool:
        rate, nh, _ = cpu_prefill_rate(plan_bytes, wl, nh, T, pool, cores)
    return {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{nh} (layer, head) states of request 0, a {T}-token chunk each (reconstruct, fp64 chunk "
                      f"form, requantize), split over {cores} spawned processes; tokens/s of a token through all "
                      f"{wl.n_layers * wl.n_heads} heads, time = slowest process"}


def _oracle_calib_layer(payload):
    """Oracle calibration statistics of one layer (all its heads)."""
    from oracle import model
    from quantized_recurrent_state_b200 import synth
    wname, l = payload
    wl = synth.workloads()[wname]
    S0 = synth.initial_states(wl, wl.calib_seed, wl.calib_req, layers=[l])
    alpha = synth.gates(wl, wl.calib_seed)
    steps = [synth.step_inputs(wl, wl.calib_seed, wl.calib_req, t, alpha=alpha, layers=[l])
             for t in range(wl.calib_steps)]
    return model.calibrate(wl.mode, wl.d, 1, wl.n_heads, S0, steps, wl.bits)


def _n_cores():
    return max(1, min(os.cpu_count() or 1, 32))


def oracle_pool(cores: int):
    """`cores` spawned worker processes, each with one BLAS thread, so that
    the oracle uses exactly `cores` threads."""
    import multiprocessing as mp
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"   # read by the workers' numpy at import
    return mp.get_context("spawn").Pool(cores)


def cpu_sample_rate(plan_bytes, wl, heads_per_step, t, pool, cores):
    """Head-steps/s of the oracle over one sample: heads split across the
    worker processes; the step time is the slowest worker's stepping time."""
    heads = [(l, h) for l in range(wl.n_layers) for h in range(wl.n_heads)][:heads_per_step]
    chunks = [heads[i::cores] for i in range(cores)]
    secs = pool.map(_oracle_sample, [(plan_bytes, wl.name, c, t) for c in chunks if c])
    return len(heads), max(secs)


def cpu_baseline(plan_bytes, wl, budget_s=12.0):
    """The oracle, as it stands, on the host cores: a bounded sample of the
    same workload (request 0's heads in layer order, one decode step each)
    sized to about budget_s seconds of CPU work in total."""
    cores = _n_cores()
    one = [(l, h) for l in range(2) for h in range(wl.n_heads)][:16]
    with oracle_pool(1) as pool1:   # one process, one BLAS thread
        sec1 = pool1.map(_oracle_sample, [(plan_bytes, wl.name, one, 0)])[0]
    per_head = sec1 / len(one)
    heads = int(min(wl.n_layers * wl.n_heads, max(cores, budget_s / max(per_head, 1e-4))))
    with oracle_pool(cores) as pool:
        nh, sec = cpu_sample_rate(plan_bytes, wl, heads, 0, pool, cores)
    return {"value": nh / sec, "unit": "head-steps/s", "cores": cores, "host_cores": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{nh} (layer, head) states of request 0, one decode step each, split over {cores} "
                      f"spawned processes; time = slowest process's stepping time",
            "single_thread": {"value": len(one) / sec1, "unit": "head-steps/s", "cores": 1,
                              "sample": f"{len(one)} (layer, head) states of request 0, one step each, "
                                        f"one process with one BLAS thread"}}


def oracle_plan_bytes(wl, pool):
    """The workload's plan from the oracle's calibration and allocator (one
    worker per layer)."""
    from oracle import model, plan_io
    layer_stats = pool.map(_oracle_calib_layer, [(wl.name, l) for l in range(wl.n_layers)])
    stats = {k: np.concatenate([np.asarray(s[k]).reshape((1,) + np.asarray(s[k]).shape[1:])
                                if k in ("wbar", "rho") else np.asarray(s[k]) for s in layer_stats])
             for k in ("wbar", "rho", "lgate", "dist")}
    plan = model.build_plan(wl.mode, wl.d, wl.n_layers, wl.n_heads, stats, wl.bits, wl.nominal_bits,
                            wl.n_pivots, wl.horizon)
    return plan_io.write_plan(None, plan)


def run_reference_prefill(args):
    """The CPU oracle's packed prefill as the reference arm of --prefill:
    each step a bounded sample of (layer, head) states of one request, a
    PREFILL_CPU_TOKENS-token chunk each."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from quantized_recurrent_state_b200 import synth
    wl = workload_of(args, synth)
    cores = _n_cores()
    T = PREFILL_CPU_TOKENS
    with oracle_pool(cores) as pool:
        plan_bytes = oracle_plan_bytes(wl, pool)
        for _ in range(args.warmup):
            cpu_prefill_rate(plan_bytes, wl, cores, T, pool, cores)
        tot_tok, tot_s = 0.0, 0.0
        for _ in range(args.steps):
            rate, nh, sec = cpu_prefill_rate(plan_bytes, wl, cores, T, pool, cores)
            tot_tok += rate * sec
            tot_s += sec
    value = tot_tok / tot_s
    sample = (f"each step: {cores} (layer, head) states of one request, a {T}-token chunk each, split over "
              f"{cores} spawned processes (time = slowest process); tokens/s of a token through all "
              f"{wl.n_layers * wl.n_heads} heads")
    out = {"impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": {**prefill_config(wl, args.batch, args.prefill, args.gpus), "variant": "oracle (CPU)"},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_reference(args):
    """The CPU oracle as the reference arm: same metric and workload, each
    step a bounded sample of (layer, head) states of one request."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from quantized_recurrent_state_b200 import synth
    wl = workload_of(args, synth)
    cores = _n_cores()
    with oracle_pool(cores) as pool:
        plan_bytes = oracle_plan_bytes(wl, pool)
        heads_per_step = 4 * cores
        for i in range(args.warmup):
            cpu_sample_rate(plan_bytes, wl, heads_per_step, i, pool, cores)
        tot_h, tot_s = 0, 0.0
        for i in range(args.steps):
            nh, sec = cpu_sample_rate(plan_bytes, wl, heads_per_step, i, pool, cores)
            tot_h += nh
            tot_s += sec
    value = tot_h / tot_s
    sample = (f"each step: {heads_per_step} (layer, head) states of one request stepped once, split over "
              f"{cores} spawned processes (time = slowest process)")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "head-steps/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic",
           "config": {**workload_config(wl, args.batch, args.gpus), "variant": "oracle (CPU)"},
           "cpu_baseline": {"value": value, "unit": "head-steps/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "head-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.prefill:
        (run_reference_prefill if args.impl == "reference" else run_prefill)(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_product(args)


if __name__ == "__main__":
    main()
