"""Long-horizon drift of the packed state against the FP32-state recurrence.

    python -m quantized_recurrent_state_b200.drift [--steps 8192] [--every 256]

STEPQuant paper digest (vibe-research), 背景与动机: quantization error is
written back every step and propagates as E_t = A_t E_{t-1} + eps_t, so a
long-lived state can carry it for many steps.  This study runs, on the GPU,
the packed path (fused kernel) and the FP32-state kernel side by side from
the same S_0 on the drift workload (4 requests x 8 GDN heads, d = 128,
half-lives 1,000-20,000 steps) for the plans: nominal 4-bit over {2,4,6,8} and nominal 6-bit over {4,6,8}
(calibrated, with pivots), uniform INT8 with the STEPQuant fit, and the
pages' baselines, uniform INT8 / INT6 / INT4 with the ordinary per-row
absmax quantizer (实验).  It reports the relative readout error every step and the
relative state error every `every` steps, and at a few steps checks the
recorded error recursion: with S~_t the fp32 update of the reconstructed
state, eps_t = S^_t - S~_t and A_t E_{t-1} the update of E_{t-1} with v = 0,
|E_t - A_t E_{t-1} - eps_t| / |E_t| must be at fp32 rounding level.

All arithmetic of the step runs in libstepq; torch only reduces the error
norms for the report.
"""
from __future__ import annotations

import argparse
import json
import math

import numpy as np


KINDS = ("nominal4", "nominal6", "int8", "absmax8", "absmax6", "absmax4")


def plan_for(stepq, synth, wl, kind, device):
    """GPU calibration + the library planner; the uniform baselines are
    fixed plans from the library's uniform-plan builder."""
    import torch
    L, H, D = wl.n_layers, wl.n_heads, wl.d
    if kind == "int8":
        return stepq.Plan.build_uniform(0, L, H, D, 8, stepq.QUANT_DUAL_AXIS, wl.horizon)
    if kind.startswith("absmax"):
        return stepq.Plan.build_uniform(0, L, H, D, int(kind[6:]), stepq.QUANT_ABSMAX, wl.horizon)
    bits, nominal = ((2, 4, 6, 8), 4.0) if kind == "nominal4" else ((4, 6, 8), 6.0)
    host = stepq.Plan.build_uniform(0, L, H, D, 8, stepq.QUANT_DUAL_AXIS, wl.horizon)
    n = wl.calib_req
    ctx = stepq.Context(host, n)
    alpha = synth.gates(wl, wl.calib_seed)
    om = torch.zeros((L, H, D), dtype=torch.float64, device=device)
    ls = torch.zeros_like(om)
    S = synth.initial_states_torch(wl, wl.calib_seed, n, 0, device)
    slots = torch.arange(n, dtype=torch.int32, device=device)
    steps = [synth.step_inputs_torch(wl, wl.calib_seed, n, t, alpha, device) for t in range(wl.calib_steps)]
    for st in steps:
        ctx.calib_accumulate(n, 0, L, st["q"], st["k"], st["alpha"], st["beta"], om, ls)
    ctx.sync()
    omega = om.cpu().numpy() / (wl.calib_steps * n)
    lmean = ls.cpu().numpy() / (wl.calib_steps * n)
    wbar = np.maximum(omega / omega.mean(axis=2, keepdims=True), 1e-12).astype(np.float32)
    dist = torch.zeros((L, H, D, len(bits)), dtype=torch.float64, device=device)
    o = torch.zeros((n, L, H, D), dtype=torch.float32, device=device)
    snaps = 0
    for t, st in enumerate(steps):
        ctx.fp32_decode_step(S, slots, n, 0, L, st["q"], st["k"], st["v"], st["alpha"], st["beta"], o)
        if (t + 1) % 8 == 0:
            ctx.calib_distortion(n, 0, L, S, torch.from_numpy(wbar).to(device), list(bits), dist)
            snaps += 1
    ctx.sync()
    ctx.close()
    d = dist.cpu().numpy() / (snaps * n)
    return stepq.Plan.build(0, L, H, D, list(bits), nominal, wl.n_pivots, wl.horizon,
                            lmean.mean(axis=2).reshape(-1), d.sum(axis=2).reshape(-1, len(bits)), wbar.reshape(-1))


def run(steps: int = 8192, every: int = 256, checks: int = 4, device: str = "cuda", kinds=KINDS):
    import torch

    from quantized_recurrent_state_b200 import build as qbuild
    qbuild.build()
    from quantized_recurrent_state_b200 import stepq, synth

    wl = synth.workloads()["drift"]
    L, H, D, n = wl.n_layers, wl.n_heads, wl.d, wl.n_req
    alpha = synth.gates(wl, wl.seed)
    out = {"workload": f"{n} requests x {H} GDN heads, d={D}, half-lives {wl.halflife[0]:g}-{wl.halflife[1]:g}",
           "steps": steps, "plans": {}}
    check_at = set(int(x) for x in np.linspace(every, steps, checks))
    for kind in kinds:
        plan = plan_for(stepq, synth, wl, kind, device)
        ctx = stepq.Context(plan, n)
        slots = torch.arange(n, dtype=torch.int32, device=device)
        pool = torch.zeros(n * plan.slot_bytes, dtype=torch.uint8, device=device)
        S0 = synth.initial_states_torch(wl, wl.seed, n, 0, device)
        ctx.requant_pack(pool, slots, n, 0, L, S0)
        S32 = S0.clone()
        Sh = torch.empty_like(S0)
        o_q = torch.zeros((n, L, H, D), dtype=torch.float32, device=device)
        o_f = torch.zeros_like(o_q)
        ro_err, st_err, rec_res = [], [], []
        prev_hat = None
        for t in range(steps):
            inp = synth.step_inputs_torch(wl, wl.seed, n, t, alpha, device)
            check = (t + 1) in check_at
            if check:
                ctx.unpack(pool, slots, n, 0, L, Sh)
                ctx.sync()
                prev_hat = Sh.clone()
                E_prev = prev_hat - S32
            ctx.decode_step_fused(pool, slots, n, 0, L, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o_q)
            ctx.fp32_decode_step(S32, slots, n, 0, L, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o_f)
            ctx.sync()
            ro_err.append(float((o_q - o_f).norm() / o_f.norm()))
            if (t + 1) % every == 0 or check:
                ctx.unpack(pool, slots, n, 0, L, Sh)
                ctx.sync()
                st_err.append((t + 1, float((Sh - S32).norm() / S32.norm())))
            if check:
                # S~_t: fp32 update of the reconstructed S^_{t-1}; A_t E_{t-1}: update with v = 0
                Stil = prev_hat.clone()
                AE = E_prev.clone()
                scratch = torch.zeros_like(o_q)
                ctx.fp32_decode_step(Stil, slots, n, 0, L, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                     scratch)
                ctx.fp32_decode_step(AE, slots, n, 0, L, inp["q"], inp["k"], torch.zeros_like(inp["v"]),
                                     inp["alpha"], inp["beta"], scratch)
                ctx.sync()
                E_t = Sh - S32
                eps = Sh - Stil
                rec_res.append((t + 1, float((E_t - AE - eps).norm() / E_t.norm())))
        ctx.close()
        out["plans"][kind] = {
            "bits_per_value": plan.info.bits_per_value,
            "bits_per_value_s16": plan.info.bits_per_value_s16,
            "readout_rel_err_mean": float(np.mean(ro_err)),
            "readout_rel_err_last_256": float(np.mean(ro_err[-256:])),
            "readout_rel_err_max": float(np.max(ro_err)),
            "state_rel_err": st_err,
            "error_recursion_residual": rec_res,
        }
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--steps", type=int, default=8192)
    ap.add_argument("--every", type=int, default=256)
    args = ap.parse_args()
    print(json.dumps(run(args.steps, args.every)))


if __name__ == "__main__":
    main()
