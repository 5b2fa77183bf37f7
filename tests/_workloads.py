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
    for that head (None: expect exact).  Returns (n_codes, n_excused, n_bad,
    max rel diff of r/c)."""
    n_codes = n_excused = n_bad = 0
    worst_scale = 0.0
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
            zg, hg, r_g, c_g = model.unpack_head(pv.mode, pv.D, rw, rg)
            zo, ho, r_o, c_o = model.unpack_head(pv.mode, pv.D, rw, ro)
            tie = ties[(l, h)]
            mism = (zg != zo) | (hg != ho)
            if tie is not None:
                excused = mism & (tie != 0)
            else:
                excused = np.zeros_like(mism)
            n_excused += int(excused.sum())
            n_bad += int((mism & ~excused).sum())
            for a, b in ((r_g, r_o), (c_g, c_o)):
                d = np.abs(a.astype(np.float64) - b.astype(np.float64))
                den = np.maximum(np.abs(b.astype(np.float64)), 1e-30)
                if tie is not None:
                    pass
                worst_scale = max(worst_scale, float(np.max(d / den)))
    return n_codes, n_excused, n_bad, worst_scale
