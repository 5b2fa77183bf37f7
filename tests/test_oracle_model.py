"""Plan- and pool-level oracle checks on the tiny GDN and a small KDA workload.

Pins: the planner respects the budget and pivot count exactly; the packed
trajectory stays close to the FP32-state trajectory (quantization error only);
lockstep over the pool reuses the head-level functions pinned elsewhere.
"""
import numpy as np

from oracle import allocator, model, plan_io
from quantized_recurrent_state_b200 import synth


def _calib_plan(wl, n_layers=None):
    L = wl.n_layers if n_layers is None else n_layers
    S0 = synth.initial_states(wl, wl.calib_seed, wl.calib_req, layers=range(L))
    alpha = synth.gates(wl, wl.calib_seed)
    steps = [synth.step_inputs(wl, wl.calib_seed, wl.calib_req, t, alpha=alpha, layers=range(L))
             for t in range(wl.calib_steps)]
    stats = model.calibrate(wl.mode, wl.d, L, wl.n_heads, S0, steps, wl.bits)
    return model.build_plan(wl.mode, wl.d, L, wl.n_heads, stats, wl.bits, wl.nominal_bits,
                            wl.n_pivots, wl.horizon)


def test_tiny_plan_budget_and_pivots(tmp_path):
    wl = synth.workloads()["tiny_gdn"]
    plan = _calib_plan(wl)
    w = plan["widths"]
    assert (w == 16).sum() == wl.n_pivots
    nonpiv = w[w != 16]
    assert nonpiv.sum() <= allocator.budget_cap(wl.nominal_bits, nonpiv.size)
    assert set(nonpiv.tolist()) <= set(wl.bits)
    data = plan_io.write_plan(str(tmp_path / "tiny.plan"), plan)
    back = plan_io.read_plan(data)
    assert np.array_equal(back["widths"], w)
    assert np.all(back["rho"] > 0) and np.all(np.isfinite(back["rho"]))


def test_tiny_packed_trajectory_tracks_fp32():
    wl = synth.workloads()["tiny_gdn"]
    plan = _calib_plan(wl)
    pv = model.PlanView(plan)
    S0 = synth.initial_states(wl, wl.seed, 1)
    pool = np.zeros((1, pv.slot_bytes), np.uint8)
    for h in range(wl.n_heads):
        pv.quantize_into(pool[0], 0, h, S0[0, 0, h])
    S_ref = S0[0, 0].copy()
    alpha = synth.gates(wl, wl.seed)
    rel = []
    for t in range(wl.steps):
        inp = synth.step_inputs(wl, wl.seed, 1, t, alpha=alpha)
        for h in range(wl.n_heads):
            a = inp["alpha"][0, 0, h]
            o, tie, S, w = pv.step(pool[0], 0, h, inp["q"][0, 0, h], inp["k"][0, 0, h],
                                   inp["v"][0, 0, h], a, inp["beta"][0, 0, h])
            from oracle import core
            o_ref = core.step_fp32(S_ref[h], inp["q"][0, 0, h], inp["k"][0, 0, h],
                                   inp["v"][0, 0, h], a, inp["beta"][0, 0, h])
            rel.append(np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref))
    # 2..6-bit codes + one FP16 head: a few percent of readout error at most
    assert np.median(rel) < 0.1, np.median(rel)


def test_kda_small_plan_lagrangian():
    wl = synth.Workload("kda_small", 1, 1, 2, 16, 1, 16, (4, 6, 8), 6.0, 3, (4.0, 2000.0), 11, 21)
    plan = _calib_plan(wl)
    w = plan["widths"]
    assert w.size == 2 * 16 and (w == 16).sum() == 3
    nonpiv = w[w != 16]
    assert nonpiv.sum() <= allocator.budget_cap(6.0, nonpiv.size)
    pv = model.PlanView(plan)
    S0 = synth.initial_states(wl, wl.seed, 1)
    pool = np.zeros((1, pv.slot_bytes), np.uint8)
    for h in range(2):
        pv.quantize_into(pool[0], 0, h, S0[0, 0, h])
        Sh = pv.reconstruct(pool[0], 0, h)
        assert np.linalg.norm(Sh - S0[0, 0, h]) / np.linalg.norm(S0[0, 0, h]) < 0.05
