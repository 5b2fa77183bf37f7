"""Shared test helpers: oracle-built plans for the named workloads and the
lockstep comparison of the CUDA path against the oracle.

The plan of each workload comes from the oracle's own calibration and
allocator; the library only parses it (so a parity failure cannot hide in a
shared planner).
"""
from __future__ import annotations

import functools

import numpy as np

from oracle import model, plan_io
from quantized_recurrent_state_b200 import synth


@functools.lru_cache(maxsize=None)
def oracle_plan(name: str, n_layers: int = None, n_pivots: int = None, d: int = None, scale_bits: int = 32):
    """(plan dict, plan bytes, Workload) for a workload, optionally sliced."""
    wl = synth.workloads()[name]
    if n_layers is not None or n_pivots is not None:
        wl = synth.Workload(**{**wl.__dict__, "n_layers": n_layers or wl.n_layers,
                               "n_pivots": wl.n_pivots if n_pivots is None else n_pivots})
    L = wl.n_layers
    S0 = synth.initial_states(wl, wl.calib_seed, wl.calib_req)
    alpha = synth.gates(wl, wl.calib_seed)
    steps = [synth.step_inputs(wl, wl.calib_seed, wl.calib_req, t, alpha=alpha) for t in range(wl.calib_steps)]
    stats = model.calibrate(wl.mode, wl.d, L, wl.n_heads, S0, steps, wl.bits)
    plan = model.build_plan(wl.mode, wl.d, L, wl.n_heads, stats, wl.bits, wl.nominal_bits, wl.n_pivots,
                            wl.horizon, scale_bits=scale_bits)
    data = plan_io.write_plan(None, plan)
    return plan, data, wl, stats


@functools.lru_cache(maxsize=None)
def uniform_plan(name: str, bits: int, quantizer: int, n_layers: int = None, scale_bits: int = 32):
    """(plan dict, plan bytes, Workload) of a baseline plan (every unit at
    `bits`, no pivots) over a workload's shape."""
    wl = synth.workloads()[name]
    wl = synth.Workload(**{**wl.__dict__, "n_layers": n_layers or wl.n_layers, "n_pivots": 0})
    plan = model.uniform_plan(wl.mode, wl.d, wl.n_layers, wl.n_heads, bits, quantizer, wl.horizon,
                              scale_bits=scale_bits)
    return plan, plan_io.write_plan(None, plan), wl, None


def compare_records(pv: model.PlanView, gpu_slot: np.ndarray, ora_slot: np.ndarray, ties: dict):
    """Compare every record of one slot.  ties[(l, h)] = the oracle's tie map
    for that head (None: expect exact).

    Codes must match except where the tie map excuses them; the row factors r
    must match bit for bit (they depend on S_t alone); the column factors c
    must match bit for bit except in columns whose initial codes had a tie
    (the refinement then sums other codes).  Returns (n_codes, n_excused,
    n_bad, n_scale_bad) where n_scale_bad counts r and c values that differ
    outside those columns."""
    n_codes = n_excused = n_bad = n_scale_bad = 0
    for l in range(pv.L):
        for h in range(pv.H):
            if (l, h) not in ties:
                continue
            rg = pv.record(gpu_slot, l, h)
            ro = pv.record(ora_slot, l, h)
            rw = pv.rw(l, h)
            n_codes += pv.D * pv.D
            if np.array_equal(rg, ro):
                continue
            zg, hg, r_g, c_g = model.unpack_head(pv.mode, pv.D, rw, rg, pv.scale_bits)
            zo, ho, r_o, c_o = model.unpack_head(pv.mode, pv.D, rw, ro, pv.scale_bits)
            tie = ties[(l, h)]
            mism = (zg != zo) | (hg != ho)
            excused = mism & (tie != 0) if tie is not None else np.zeros_like(mism)
            n_excused += int(excused.sum())
            n_bad += int((mism & ~excused).sum())
            n_scale_bad += int((r_g.view(np.uint32) != r_o.view(np.uint32)).sum())
            tie_cols = ((tie & 2) != 0).any(axis=0) if tie is not None else np.zeros(pv.D, bool)
            n_scale_bad += int(((c_g.view(np.uint32) != c_o.view(np.uint32)) & ~tie_cols).sum())
    return n_codes, n_excused, n_bad, n_scale_bad


def reconstruction_gap(pv: model.PlanView, gpu_slot: np.ndarray, ora_slot: np.ndarray, heads, excused=None):
    """Largest |S_hat_gpu - S_hat_oracle| / (1e-5 + 1e-4 |S_hat_oracle|) over the
    reconstructed states of `heads` [(l, h)], the stated tolerance on
    reconstructed states (<= 1 passes); elements whose codes were excused as
    rounding ties are left out when `excused` maps (l, h) to the tie map."""
    worst = 0.0
    for (l, h) in heads:
        a = pv.reconstruct(gpu_slot, l, h).astype(np.float64)
        b = pv.reconstruct(ora_slot, l, h).astype(np.float64)
        r = np.abs(a - b) / (1e-5 + 1e-4 * np.abs(b))
        if excused is not None and excused.get((l, h)) is not None:
            r = np.where(excused[(l, h)] != 0, 0.0, r)
        worst = max(worst, float(r.max()))
    return worst
