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


# --------------------------------------------------------------------------
# calibration statistics (方法-2 row impact, 方法-1 mean log gate and d_u(b))
# --------------------------------------------------------------------------

from oracle import core  # noqa: E402

_rng = np.random.default_rng(777)


def _explicit_A(alpha, beta, k):
    """A_t = (I - beta k k^T) Diag(alpha) as a dense fp64 matrix."""
    D = k.size
    k64 = k.astype(np.float64)
    return (np.eye(D) - np.float64(beta) * np.outer(k64, k64)) @ np.diag(alpha.astype(np.float64))


def test_calib_accumulate_is_A_transpose_q():
    # omega_i += g_i^2 with g = A_t^T q_t, A_t built as an explicit matrix; per-row gates make
    # A_t^T q differ from A_t q and from a version without the gate
    D = 128
    for kda in (False, True):
        q = _rng.standard_normal(D).astype(np.float32)
        n = _rng.standard_normal(D)
        k = (n / np.linalg.norm(n)).astype(np.float32)
        alpha = (_rng.uniform(0.3, 1.0, D) if kda else np.full(D, _rng.uniform(0.3, 1.0))).astype(np.float32)
        beta = np.float32(_rng.uniform(0.2, 1.0))
        om = np.zeros(D)
        ls = np.zeros(D)
        core.calib_accumulate(q, k, alpha, beta, om, ls)
        g = _explicit_A(alpha, beta, k).T @ q.astype(np.float64)
        assert np.allclose(om, g * g, rtol=1e-12, atol=1e-300)
        assert np.allclose(ls, np.log(alpha.astype(np.float64)), rtol=1e-15, atol=0)
        if kda:
            g_wrong = _explicit_A(alpha, beta, k) @ q.astype(np.float64)
            assert not np.allclose(om, g_wrong * g_wrong, rtol=1e-3)


def test_calibrate_statistics_from_explicit_matrices():
    # tiny GDN workload: omega from explicit A_t^T q over every step and request, its
    # normalisation wbar = omega / mean(omega) per head (mean 1), rho = wbar^(-1/4), and
    # l_u = the mean log gate of the head
    wl = synth.workloads()["tiny_gdn"]
    L, H, D = wl.n_layers, wl.n_heads, wl.d
    S0 = synth.initial_states(wl, wl.calib_seed, wl.calib_req)
    alpha = synth.gates(wl, wl.calib_seed)
    steps = [synth.step_inputs(wl, wl.calib_seed, wl.calib_req, t, alpha=alpha) for t in range(wl.calib_steps)]
    stats = model.calibrate(wl.mode, D, L, H, S0, steps, wl.bits)
    omega = np.zeros((L, H, D))
    lsum = np.zeros((L, H))
    cnt = 0
    for st in steps:
        for n in range(wl.calib_req):
            for l in range(L):
                for h in range(H):
                    a = np.full(D, st["alpha"][n, l, h], np.float32)
                    g = _explicit_A(a, st["beta"][n, l, h], st["k"][n, l, h]).T @ st["q"][n, l, h].astype(np.float64)
                    omega[l, h] += g * g
                    lsum[l, h] += np.log(np.float64(a[0]))
        cnt += wl.calib_req
    omega /= cnt
    wbar_ref = np.maximum(omega / omega.mean(axis=2, keepdims=True), 1e-12)
    wbar = stats["wbar"].astype(np.float64)
    assert np.allclose(wbar, wbar_ref, rtol=1e-6)
    assert np.allclose(wbar.mean(axis=2), 1.0, rtol=1e-6)
    rho = stats["rho"].astype(np.float64)
    assert np.allclose(rho ** 4 * wbar, 1.0, rtol=5e-7)
    assert np.allclose(stats["lgate"], (lsum / cnt).reshape(-1), rtol=1e-12)


def test_distortion_rows_axis_and_closed_cases():
    D = 16
    ones = np.ones(D, np.float32)
    # (1) per-row aggregation: err_rows[i] = sum_j (S_hat_ij - S_ij)^2 of that row, on a state whose
    #     rows and columns differ in scale by orders of magnitude (a column sum would not match)
    S = (_rng.standard_normal((D, D)) * np.logspace(-2, 2, D)[:, None] * np.logspace(1, -1, D)[None, :]).astype(np.float32)
    for b in (2, 4, 6, 8):
        rw = np.full(D, b, np.int32)
        z, h, r, c, _ = core.quantize(D, rw, ones, ones, S)
        Sh = core.reconstruct(D, rw, z, h, r, c).astype(np.float64)
        err = core.distortion_rows(D, b, ones, ones, S)
        row = ((Sh - S.astype(np.float64)) ** 2).sum(axis=1)
        assert np.allclose(err, row, rtol=1e-12, atol=0)
        assert not np.allclose(err, ((Sh - S.astype(np.float64)) ** 2).sum(axis=0), rtol=1e-3)
    # (2) constant magnitude at b = 2 (codes +-1, c = 1): exact reconstruction, zero error
    Sc = (np.where(_rng.uniform(size=(D, D)) < 0.5, -1.0, 1.0) * 2.0 ** _rng.integers(-3, 4, (D, 1))).astype(np.float32)
    assert np.all(core.distortion_rows(D, 2, ones, ones, Sc) == 0.0)
    # (3) scaling the head by 2^k scales every row error by 4^k exactly
    e1 = core.distortion_rows(D, 6, ones, ones, S)
    e2 = core.distortion_rows(D, 6, ones, ones, (S * np.float32(8.0)).astype(np.float32))
    assert np.array_equal(e2, e1 * 64.0)
