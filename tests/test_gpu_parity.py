"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Lockstep protocol: at every step the oracle starts from the records the GPU
holds, so one excused rounding tie cannot propagate.  Packed codes must be
bit-exact except codes whose oracle pre-rounding value lies within 1e-6
relative of a .5 boundary (or whose column's initial codes had such a tie);
those are counted and must stay <= 1e-5 of all codes.  Readouts must satisfy
|o_gpu - o_ref| <= 1e-5 + 1e-4 |o_ref|.
"""
import numpy as np
import pytest

from oracle import core, model
from quantized_recurrent_state_b200 import synth
from tests._workloads import compare_records, oracle_plan, reconstruction_gap, uniform_plan

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-4, 1e-5


@pytest.fixture(scope="module")
def stepq():
    from quantized_recurrent_state_b200 import build as qbuild
    qbuild.build()
    from quantized_recurrent_state_b200 import stepq as s
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return s


def _close(g, r):
    return np.abs(g - r) <= ATOL + RTOL * np.abs(r)


def _inputs_to_dev(inp):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in inp.items()}


class Run:
    """A GPU pool for a workload plus an oracle view of the same plan."""

    def __init__(self, stepq, name, n_req, n_layers=None, n_pivots=None, extra_slots=3, chunk=2, uniform=None,
                 scale_bits=32, step_kernel=0):
        if uniform is None:
            self.plan, data, self.wl, _ = oracle_plan(name, n_layers, n_pivots, scale_bits=scale_bits)
        else:  # (bits, quantizer): a baseline plan over the workload's shape
            self.plan, data, self.wl, _ = uniform_plan(name, uniform[0], uniform[1], n_layers, scale_bits=scale_bits)
        self.pv = model.PlanView(self.plan)
        self.P = stepq.Plan.from_bytes(data)
        self.n_req = n_req
        self.n_slots = n_req + extra_slots
        rng = np.random.default_rng(7)
        self.slots = rng.permutation(self.n_slots)[:n_req].astype(np.int32)
        self.slots_t = torch.from_numpy(self.slots).cuda()
        self.ctx = stepq.Context(self.P, self.n_slots, chunk_layers=chunk)
        self.ctx.set_step_kernel(step_kernel)
        self.pool = torch.zeros(self.n_slots * self.P.slot_bytes, dtype=torch.uint8, device="cuda")
        self.L = self.wl.n_layers
        self.alpha = synth.gates(self.wl, self.wl.seed)

    def slot_bytes_host(self, n):
        sb = self.P.slot_bytes
        s = int(self.slots[n])
        return self.pool[s * sb:(s + 1) * sb].cpu().numpy()

    def pack_initial(self):
        S0 = synth.initial_states(self.wl, self.wl.seed, self.n_req)
        self.ctx.requant_pack(self.pool, self.slots_t, self.n_req, 0, self.L, torch.from_numpy(S0).cuda())
        self.ctx.sync()
        return S0

    def step(self, t, fused=False, ws=None):
        inp = synth.step_inputs(self.wl, self.wl.seed, self.n_req, t, alpha=self.alpha)
        d = _inputs_to_dev(inp)
        o = torch.zeros_like(d["q"])
        if fused:
            self.ctx.decode_step_fused(self.pool, self.slots_t, self.n_req, 0, self.L, d["q"], d["k"], d["v"],
                                       d["alpha"], d["beta"], o)
        else:
            if ws is None:
                ws = torch.empty(self.ctx.workspace_bytes(self.n_req, self.L) // 4, dtype=torch.float32,
                                 device="cuda")
            self.ctx.decode_step(self.pool, self.slots_t, self.n_req, 0, self.L, d["q"], d["k"], d["v"],
                                 d["alpha"], d["beta"], o, ws)
        self.ctx.sync()
        return inp, o.cpu().numpy()


@pytest.mark.parametrize("name,n,steps,kw", [("qwen_layer", 3, 64, {}),
                                              ("kda_rows", 2, 24, {"n_layers": 1, "n_pivots": 8})])
def test_free_running_trajectory(stepq, name, n, steps, kw):
    """The free-running comparison beside the lockstep one: the GPU (fused
    step) and the oracle each step their own records from the same S_0, with
    no resynchronisation.  Until the oracle meets a rounding tie (a non-zero
    tie map) the two trajectories must stay identical bit for bit, records and
    readouts; after a tie the run only reports the step of the first
    difference and how far the readouts have drifted."""
    run = Run(stepq, name, n, **kw)
    S0 = run.pack_initial()
    pv = run.pv
    ora, tie_step = {}, None
    for r in range(n):
        slot = np.zeros(run.P.slot_bytes, np.uint8)
        for l in range(pv.L):
            for h in range(pv.H):
                if pv.quantize_into(slot, l, h, S0[r, l, h]).any():
                    tie_step = -1 if tie_step is None else tie_step
        ora[r] = slot
    first_diff, worst_o = None, 0.0
    for t in range(-1, steps):
        if t >= 0:
            inp, o = run.step(t, fused=True)
        for r in range(n):
            if t >= 0:
                for l in range(pv.L):
                    for h in range(pv.H):
                        o_ref, tie, _, _ = pv.step(ora[r], l, h, inp["q"][r, l, h], inp["k"][r, l, h], inp["v"][r, l, h],
                                                   inp["alpha"][r, l, h], inp["beta"][r, l, h])
                        if tie.any() and tie_step is None:
                            tie_step = t
                        if not np.array_equal(o[r, l, h], o_ref):
                            first_diff = t if first_diff is None else first_diff
                        scale = max(1e-30, float(np.max(np.abs(o_ref))))
                        worst_o = max(worst_o, float(np.max(np.abs(o[r, l, h] - o_ref))) / scale)
            if not np.array_equal(run.slot_bytes_host(r), ora[r]):
                first_diff = t if first_diff is None else first_diff
        if tie_step is None:
            assert first_diff is None, (t, "trajectories differ before any rounding tie")
    print(f"free-running {name}: {steps} steps, first tie {tie_step}, first difference {first_diff}, "
          f"worst readout difference {worst_o:.3g} of the head's largest readout")


def _lockstep(stepq, name, n_req, steps, check, n_layers=None, n_pivots=None, fused=False, heads=None,
              uniform=None, scale_bits=32, step_kernel=0):
    run = Run(stepq, name, n_req, n_layers, n_pivots, uniform=uniform, scale_bits=scale_bits, step_kernel=step_kernel)
    S0 = run.pack_initial()
    pv = run.pv
    tot_codes = tot_exc = tot_bad = 0
    # packing of S_0
    for n in check:
        g = run.slot_bytes_host(n)
        ora = np.zeros_like(g)
        ties = {}
        for l in range(pv.L):
            for h in range(pv.H):
                if heads is not None and h not in heads:
                    continue
                ties[(l, h)] = pv.quantize_into(ora, l, h, S0[n, l, h])
        c, e, b, sb = compare_records(pv, g, ora, ties)
        tot_codes += c; tot_exc += e; tot_bad += b
        assert sb == 0, ("scales", n, sb)
    assert tot_bad == 0
    worst_o = worst_s = 0.0
    for t in range(steps):
        prev = {n: run.slot_bytes_host(n) for n in check}
        inp, o = run.step(t, fused=fused)
        for n in check:
            g = run.slot_bytes_host(n)
            ora = prev[n].copy()
            ties = {}
            for l in range(pv.L):
                for h in range(pv.H):
                    if heads is not None and h not in heads:
                        continue
                    o_ref, tie, S, w = pv.step(ora, l, h, inp["q"][n, l, h], inp["k"][n, l, h], inp["v"][n, l, h],
                                               inp["alpha"][n, l, h], inp["beta"][n, l, h])
                    ties[(l, h)] = tie
                    ok = _close(o[n, l, h], o_ref)
                    assert ok.all(), (t, n, l, h, np.max(np.abs(o[n, l, h] - o_ref)))
                    worst_o = max(worst_o, float(np.max(np.abs(o[n, l, h] - o_ref) / (ATOL + RTOL * np.abs(o_ref)))))
            c, e, b, sb = compare_records(pv, g, ora, ties)
            tot_codes += c; tot_exc += e; tot_bad += b
            assert b == 0, (t, n, b)
            assert sb == 0, ("scales", t, n, sb)
            if t % 8 == 0 or t == steps - 1:  # reconstructed states (1e-5 + 1e-4 relative)
                gap = reconstruction_gap(pv, g, ora, list(ties), ties)
                assert gap <= 1.0, (t, n, gap)
                worst_s = max(worst_s, gap)
    print(f"{name}: codes {tot_codes}, tie-excused {tot_exc}, bad {tot_bad}, worst o/tol {worst_o:.3g}, "
          f"worst S_hat/tol {worst_s:.3g}")
    assert tot_exc <= 1e-5 * tot_codes
    return run


def test_tiny_gdn_pack_and_unpack(stepq):
    run = Run(stepq, "tiny_gdn", 1)
    S0 = run.pack_initial()
    pv = run.pv
    g = run.slot_bytes_host(0)
    ora = np.zeros_like(g)
    for h in range(pv.H):
        pv.quantize_into(ora, 0, h, S0[0, 0, h])
    assert np.array_equal(g, ora)
    Sh = torch.zeros((1, 1, pv.H, pv.D, pv.D), dtype=torch.float32, device="cuda")
    run.ctx.unpack(run.pool, run.slots_t, 1, 0, 1, Sh)
    run.ctx.sync()
    Sh = Sh.cpu().numpy()
    for h in range(pv.H):
        assert np.array_equal(Sh[0, 0, h], pv.reconstruct(ora, 0, h))


@pytest.mark.parametrize("fused", [False, True])
def test_tiny_gdn_lockstep_32_steps(stepq, fused):
    _lockstep(stepq, "tiny_gdn", 1, 32, check=[0], fused=fused)


@pytest.mark.parametrize("fused,step_kernel", [(True, 1), (True, 0), (False, 0)])
def test_qwen_layer_lockstep_256_steps(stepq, fused, step_kernel):
    # 64 requests x 48 heads, d = 128, nominal 6 bits over {4,6,8}, 1 pivot head;
    # the oracle follows two of the requests (96 heads) at every step; the fused
    # step (state in tensor memory, and in registers) and the two-stream step.
    _lockstep(stepq, "qwen_layer", 64, 256, check=[0, 37], fused=fused, step_kernel=step_kernel)


@pytest.mark.parametrize("name", ["qwen_pool6", "qwen_pool4"])
@pytest.mark.parametrize("fused,step_kernel", [(False, 0), (True, 1)])
def test_pool_slice_lockstep(stepq, name, fused, step_kernel):
    # a 2-layer slice of the 2,304-head pool at batch 70 (2 pivot heads), 8 steps
    _lockstep(stepq, name, 70, 8, check=[0, 69], n_layers=2, n_pivots=2, fused=fused, step_kernel=step_kernel)


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
@pytest.mark.parametrize("fused,step_kernel", [(False, 0), (True, 0), (True, 1)])
def test_absmax_baseline_lockstep(stepq, bits, fused, step_kernel):
    # uniform INT-b plans with the per-row absmax requantizer over a 2-layer
    # slice of the pool, batch 70, 6 steps; every step variant
    _lockstep(stepq, "qwen_pool6", 70, 6, check=[0, 69], n_layers=2, fused=fused,
              uniform=(bits, model.QUANT_ABSMAX), step_kernel=step_kernel)


@pytest.mark.parametrize("bits", [2, 8])
@pytest.mark.parametrize("step_kernel", [0, 1])
def test_uniform_dual_axis_lockstep(stepq, bits, step_kernel):
    # uniform INT-b with the STEPQuant fit (no pivots), fused
    _lockstep(stepq, "qwen_pool6", 70, 6, check=[0, 69], n_layers=2, fused=True, uniform=(bits, model.QUANT_DUAL_AXIS),
              step_kernel=step_kernel)


@pytest.mark.parametrize("fused,step_kernel", [(False, 0), (True, 0), (True, 1)])
def test_scale16_lockstep(stepq, fused, step_kernel):
    # calibrated nominal-6 plan with bfloat16 scale storage, 2-layer pool slice
    _lockstep(stepq, "qwen_pool6", 70, 6, check=[0, 69], n_layers=2, n_pivots=2, fused=fused, scale_bits=16,
              step_kernel=step_kernel)


def test_scale16_absmax_lockstep(stepq):
    _lockstep(stepq, "qwen_pool6", 70, 4, check=[0, 69], n_layers=2, fused=True,
              uniform=(6, model.QUANT_ABSMAX), scale_bits=16)


@pytest.mark.parametrize("name", ["gdn_d32", "gdn_d64"])
@pytest.mark.parametrize("fused", [False, True])
def test_mid_head_dims_lockstep(stepq, name, fused):
    # d = 32 and 64: every request checked, 8 steps, both step variants
    _lockstep(stepq, name, 6, 8, check=list(range(6)), fused=fused)


@pytest.mark.parametrize("name", ["gdn_d32", "gdn_d64"])
def test_mid_head_dims_absmax_scale16(stepq, name):
    _lockstep(stepq, name, 6, 4, check=[0, 5], fused=True, uniform=(4, model.QUANT_ABSMAX), scale_bits=16)


@pytest.mark.parametrize("step_kernel", [0, 1])
def test_fused_bit_identical_to_two_stream(stepq, step_kernel):
    a = Run(stepq, "qwen_layer", 9)
    b = Run(stepq, "qwen_layer", 9, step_kernel=step_kernel)
    a.pack_initial()
    b.pack_initial()
    for t in range(6):
        _, oa = a.step(t, fused=False)
        _, ob = b.step(t, fused=True)
        assert np.array_equal(oa, ob)
        assert torch.equal(a.pool, b.pool)


def test_ragged_and_empty(stepq):
    run = Run(stepq, "qwen_layer", 5, extra_slots=11)
    run.pack_initial()
    before = run.pool.clone()
    d = _inputs_to_dev(synth.step_inputs(run.wl, run.wl.seed, 5, 0, alpha=run.alpha))
    o = torch.zeros_like(d["q"])
    ws = torch.empty(run.ctx.workspace_bytes(5, 1) // 4, dtype=torch.float32, device="cuda")
    run.ctx.decode_step(run.pool, run.slots_t, 0, 0, 1, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o, ws)
    run.ctx.sync()
    assert torch.equal(run.pool, before) and float(o.abs().sum()) == 0.0
    # slots not named by the call stay untouched
    sb = run.P.slot_bytes
    untouched = sorted(set(range(run.n_slots)) - set(run.slots.tolist()))
    run.step(0)
    for s in untouched:
        assert torch.equal(run.pool[s * sb:(s + 1) * sb], before[s * sb:(s + 1) * sb])


def test_bad_slot_reports_device_error(stepq):
    run = Run(stepq, "tiny_gdn", 2)
    run.pack_initial()
    bad = torch.tensor([0, run.n_slots + 5], dtype=torch.int32, device="cuda")
    d = _inputs_to_dev(synth.step_inputs(run.wl, run.wl.seed, 2, 0, alpha=run.alpha))
    o = torch.zeros_like(d["q"])
    run.ctx.decode_step_fused(run.pool, bad, 2, 0, 1, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
    with pytest.raises(stepq.StepqError) as ei:
        run.ctx.sync()
    assert ei.value.code == stepq.EDEVICE
    run.ctx.sync()  # the word was cleared
    with pytest.raises(stepq.StepqError) as ei:
        run.ctx.decode_step_fused(run.pool[1:], run.slots_t, 2, 0, 1, d["q"], d["k"], d["v"], d["alpha"],
                                  d["beta"], o)
    assert ei.value.code == stepq.EINVAL
    with pytest.raises(stepq.StepqError) as ei:
        run.ctx.decode_step_fused(run.pool, run.slots_t, 2, 0, 2, d["q"], d["k"], d["v"], d["alpha"],
                                  d["beta"], o)
    assert ei.value.code == stepq.EINVAL


@pytest.mark.parametrize("name,n,n_layers", [("qwen_layer", 3, None), ("kda_rows", 2, 1), ("tiny_gdn", 2, None),
                                             ("gdn_d64", 3, None)])
def test_fp32_reference_kernel(stepq, name, n, n_layers):
    # the FP32-state step against the oracle's fp32 recurrence, bit for bit (same
    # definition: band-order sums, one fma per element); per-head and per-row gates,
    # d = 128, 64 and 16; 12 steps, every head
    plan, data, wl, _ = oracle_plan(name, n_layers)
    P = stepq.Plan.from_bytes(data)
    ctx = stepq.Context(P, n)
    L = wl.n_layers
    S0 = synth.initial_states(wl, wl.seed, n)
    Sd = torch.from_numpy(S0).cuda().contiguous()
    slots = torch.arange(n, dtype=torch.int32, device="cuda")
    alpha = synth.gates(wl, wl.seed)
    S_ref = S0.copy()
    for t in range(12):
        inp = synth.step_inputs(wl, wl.seed, n, t, alpha=alpha)
        d = _inputs_to_dev(inp)
        o = torch.zeros_like(d["q"])
        ctx.fp32_decode_step(Sd, slots, n, 0, L, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
        ctx.sync()
        og = o.cpu().numpy()
        for r in range(n):
            for l in range(L):
                for h in range(wl.n_heads):
                    o_ref = core.step_fp32(S_ref[r, l, h], inp["q"][r, l, h], inp["k"][r, l, h], inp["v"][r, l, h],
                                           inp["alpha"][r, l, h], inp["beta"][r, l, h])
                    assert np.array_equal(og[r, l, h], o_ref), (t, r, l, h)
    assert np.array_equal(Sd.cpu().numpy(), S_ref)


def test_calibration_kernels_match_oracle(stepq):
    plan, data, wl, stats = oracle_plan("tiny_gdn")
    P = stepq.Plan.from_bytes(data)
    D, H = wl.d, wl.n_heads
    ctx = stepq.Context(P, 1)
    alpha = synth.gates(wl, wl.calib_seed)
    om = torch.zeros((1, H, D), dtype=torch.float64, device="cuda")
    ls = torch.zeros_like(om)
    om_ref = np.zeros((1, H, D))
    ls_ref = np.zeros((1, H, D))
    for t in range(8):
        inp = synth.step_inputs(wl, wl.calib_seed, 1, t, alpha=alpha)
        d = _inputs_to_dev(inp)
        ctx.calib_accumulate(1, 0, 1, d["q"], d["k"], d["alpha"], d["beta"], om, ls)
        for h in range(H):
            core.calib_accumulate(inp["q"][0, 0, h], inp["k"][0, 0, h], inp["alpha"][0, 0, h], inp["beta"][0, 0, h],
                                  om_ref[0, h], ls_ref[0, h])
    ctx.sync()
    assert np.allclose(om.cpu().numpy(), om_ref, rtol=1e-12, atol=0)
    assert np.allclose(ls.cpu().numpy(), ls_ref, rtol=1e-12, atol=1e-300)
    S = synth.initial_states(wl, wl.seed, 1)
    wbar = stats["wbar"].reshape(1, H, D)
    dist = torch.zeros((1, H, D, 3), dtype=torch.float64, device="cuda")
    ctx.calib_distortion(1, 0, 1, torch.from_numpy(S).cuda(), torch.from_numpy(wbar).cuda(), [2, 4, 6], dist)
    ctx.sync()
    dg = dist.cpu().numpy()
    for h in range(H):
        for m, b in enumerate((2, 4, 6)):
            ref = core.distortion_rows(D, b, stats["rho"][0, h], stats["wbar"][0, h], S[0, 0, h])
            assert np.allclose(dg[0, h, :, m], ref, rtol=1e-12, atol=0)


def _full_pool_sampled(stepq, name, n, steps, n_samples, seed, reverse_slots=False, step_kernel=0):
    """The whole pool of a workload at batch n in the launch configuration the
    benchmark times: S_0 and the step inputs drawn on the device by the same
    generator, `steps` fused steps, then sampled (request, layer, head) records
    (plus heads holding FP16 units) checked against the oracle from the records
    the GPU held before the last step."""
    plan, data, wl, _ = oracle_plan(name)
    pv = model.PlanView(plan)
    P = stepq.Plan.from_bytes(data)
    ctx = stepq.Context(P, n)
    ctx.set_step_kernel(step_kernel)
    pool = torch.zeros(n * P.slot_bytes, dtype=torch.uint8, device="cuda")
    slots = torch.arange(n, dtype=torch.int32, device="cuda")
    if reverse_slots:
        slots = slots.flip(0).contiguous()
    for l in range(wl.n_layers):
        ctx.requant_pack(pool, slots, n, l, l + 1, synth.initial_states_torch(wl, wl.seed, n, l, "cuda"))
    alpha = synth.gates(wl, wl.seed)
    o = torch.zeros((n, wl.n_layers, wl.n_heads, wl.d), dtype=torch.float32, device="cuda")
    sb = P.slot_bytes
    for t in range(steps):
        inp = synth.step_inputs_torch(wl, wl.seed, n, t, alpha, "cuda")
        if t == steps - 1:
            ctx.sync()
            prev = pool.clone()
        ctx.decode_step_fused(pool, slots, n, 0, wl.n_layers, inp["q"], inp["k"], inp["v"], inp["alpha"],
                              inp["beta"], o)
    ctx.sync()
    rng = np.random.default_rng(seed)
    units = P.widths().reshape(wl.n_layers * wl.n_heads, -1)
    piv_heads = np.nonzero((units == 16).any(axis=1))[0]
    samples = [(int(rng.integers(n)), int(rng.integers(wl.n_layers)), int(rng.integers(wl.n_heads)))
               for _ in range(n_samples)]
    samples += [(n - 1, int(u) // wl.n_heads, int(u) % wl.n_heads) for u in piv_heads[:3]]
    slot_of = slots.cpu().numpy()
    n_codes = n_exc = 0
    for (r, l, h) in samples:
        slot = int(slot_of[r])
        off, nb = P.record(l, h)
        rec_prev = prev[slot * sb + off:slot * sb + off + nb].cpu().numpy()
        rec_new = pool[slot * sb + off:slot * sb + off + nb].cpu().numpy()
        x = {k: inp[k][r, l, h].cpu().numpy() for k in ("q", "k", "v", "alpha", "beta")}
        new_rec, o_ref, tie, S, w = model.step_head(pv.mode, pv.D, pv.rw(l, h), pv.rho[l, h], pv.wbar[l, h],
                                                    rec_prev, x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                                                    pv.quantizer, pv.scale_bits)
        assert _close(o[r, l, h].cpu().numpy(), o_ref).all(), (r, l, h)
        n_codes += pv.D * pv.D
        if not np.array_equal(rec_new, new_rec):
            zg, hg, rg, cg = model.unpack_head(pv.mode, pv.D, pv.rw(l, h), rec_new, pv.scale_bits)
            zo, ho, ro, co = model.unpack_head(pv.mode, pv.D, pv.rw(l, h), new_rec, pv.scale_bits)
            mism = (zg != zo) | (hg != ho)
            assert not (mism & (tie == 0)).any(), (r, l, h)
            n_exc += int(mism.sum())
            assert np.array_equal(rg.view(np.uint32), ro.view(np.uint32)), (r, l, h)
            tie_cols = ((tie & 2) != 0).any(axis=0)
            assert not ((cg.view(np.uint32) != co.view(np.uint32)) & ~tie_cols).any(), (r, l, h)
    print(f"{name} batch {n}: sampled codes {n_codes}, tie-excused {n_exc}")
    assert n_exc <= 1e-5 * n_codes


def test_layer_shard_of_full_pool_lockstep(stepq):
    # One GPU's share of a layer-sharded pool (the multi-GPU split, survey row f4):
    # the library's slice of the 48-layer nominal-6 plan (stepq_plan_slice) with its own
    # pool layout, stepped by the fused kernel, against the oracle's slice of the same
    # plan (model.slice_plan) in lockstep for 4 steps, 3 layers x 48 heads x 2 requests.
    plan, data, wl, _ = oracle_plan("qwen_pool6")
    lb, le = 20, 23
    Ps = stepq.Plan.from_bytes(data).slice(lb, le)
    pv = model.PlanView(model.slice_plan(plan, lb, le))
    assert Ps.slot_bytes == pv.slot_bytes
    assert np.array_equal(Ps.widths(), np.asarray(pv.plan["widths"], np.uint8))
    n, layers = 4, list(range(lb, le))
    ctx = stepq.Context(Ps, n)
    pool = torch.zeros(n * Ps.slot_bytes, dtype=torch.uint8, device="cuda")
    slots = torch.arange(n, dtype=torch.int32, device="cuda")
    S0 = synth.initial_states(wl, wl.seed, n, layers=layers)
    ctx.requant_pack(pool, slots, n, 0, le - lb, torch.from_numpy(S0).cuda())
    ctx.sync()
    alpha = synth.gates(wl, wl.seed)
    sb = Ps.slot_bytes
    tot = exc = 0
    for t in range(4):
        prev = pool.cpu().numpy().reshape(n, sb)
        inp = synth.step_inputs(wl, wl.seed, n, t, alpha=alpha, layers=layers)
        d = _inputs_to_dev(inp)
        o = torch.zeros_like(d["q"])
        ctx.decode_step_fused(pool, slots, n, 0, le - lb, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
        ctx.sync()
        got = pool.cpu().numpy().reshape(n, sb)
        o = o.cpu().numpy()
        for r in (0, n - 1):
            ora = prev[r].copy()
            ties = {}
            for l in range(le - lb):
                for h in range(pv.H):
                    o_ref, tie, _, _ = pv.step(ora, l, h, inp["q"][r, l, h], inp["k"][r, l, h], inp["v"][r, l, h],
                                               inp["alpha"][r, l, h], inp["beta"][r, l, h])
                    ties[(l, h)] = tie
                    assert _close(o[r, l, h], o_ref).all(), (t, r, l, h)
            c, e, b, sbad = compare_records(pv, got[r], ora, ties)
            tot += c
            exc += e
            assert b == 0 and sbad == 0, (t, r, b, sbad)
    assert exc <= 1e-5 * tot


@pytest.mark.parametrize("step_kernel", [0, 1])
def test_full_pool_sampled_heads(stepq, step_kernel):
    # the benchmark's workload: 2,304 heads, batch 70, nominal 6 bits, 32 FP16 heads; 2 steps
    _full_pool_sampled(stepq, "qwen_pool6", 70, 2, 24, 11, step_kernel=step_kernel)


@pytest.mark.parametrize("step_kernel", [0, 1])
def test_full_pool_sampled_heads_batch256(stepq, step_kernel):
    # the largest batch the benchmark sweeps: 589,824 records in one launch, an 8 GB pool,
    # slots in reverse request order
    _full_pool_sampled(stepq, "qwen_pool6", 256, 2, 16, 12, reverse_slots=True, step_kernel=step_kernel)


def test_full_pool_nominal4_sampled_heads(stepq):
    # the nominal-4 pool over {2,4,6,8} (every width in one launch), state in tensor memory
    _full_pool_sampled(stepq, "qwen_pool4", 70, 2, 24, 13, step_kernel=1)


def test_kda_full_sampled_heads(stepq):
    # 81,920 key rows (20 layers x 32 heads x 128), 512 FP16 rows, batch 128; 2 steps
    _full_pool_sampled(stepq, "kda_rows", 128, 2, 16, 5)


def test_kda_slice_lockstep_long(stepq):
    # 64 steps of a 1-layer KDA slice, every request followed, fused
    _lockstep(stepq, "kda_rows", 4, 64, check=[0, 1, 2, 3], n_layers=1, n_pivots=8, fused=True)


# ---------------------------------------------------------------------------
# per-key-row units (KDA): mixed row widths, FP16 pivot rows, per-row gates
# ---------------------------------------------------------------------------

def test_kda_slice_lockstep(stepq):
    # 2 layers x 32 heads x 128 key rows of the KDA pool, Lagrangian nominal
    # 6-bit plan over {4,6,8} with 16 FP16 rows, batch 8, 8 steps
    _lockstep(stepq, "kda_rows", 8, 8, check=[0, 7], n_layers=2, n_pivots=16)


@pytest.mark.parametrize("n_pivots,fused", [(0, True), (0, False), (512, True), (512, False)])
def test_kda_fp16_free_and_fp16_heavy_plans(stepq, n_pivots, fused):
    # The per-row step kernels run one code path for heads without FP16 rows and
    # another for heads with them (chosen per item from the step descriptor).  A
    # 1-layer KDA slice with no FP16 row sends every head down the first; with 512
    # FP16 rows over its 4,096 key rows every one of the 32 heads has some.
    plan, _, wl, _ = oracle_plan("kda_rows", n_layers=1, n_pivots=n_pivots)
    w = np.asarray(plan["widths"]).reshape(-1, wl.d)
    assert int((w == 16).any(axis=1).sum()) == (0 if n_pivots == 0 else w.shape[0])
    _lockstep(stepq, "kda_rows", 4, 6, check=[0, 3], n_layers=1, n_pivots=n_pivots, fused=fused)


def test_kda_scale16_lockstep(stepq):
    _lockstep(stepq, "kda_rows", 8, 4, check=[0, 7], n_layers=2, n_pivots=16, fused=True, scale_bits=16)


def test_kda_two_stream_equals_fused(stepq):
    a = Run(stepq, "kda_rows", 5, n_layers=2, n_pivots=16)
    b = Run(stepq, "kda_rows", 5, n_layers=2, n_pivots=16)
    a.pack_initial()
    b.pack_initial()
    for t in range(4):
        _, oa = a.step(t, fused=False)
        _, ob = b.step(t, fused=True)
        assert np.array_equal(oa, ob)
        assert torch.equal(a.pool, b.pool)


def test_kda_unpack(stepq):
    run = Run(stepq, "kda_rows", 2, n_layers=2, n_pivots=16)
    run.pack_initial()
    pv = run.pv
    Sh = torch.zeros((2, pv.L, pv.H, pv.D, pv.D), dtype=torch.float32, device="cuda")
    run.ctx.unpack(run.pool, run.slots_t, 2, 0, pv.L, Sh)
    run.ctx.sync()
    Sh = Sh.cpu().numpy()
    for n in range(2):
        g = run.slot_bytes_host(n)
        for (l, h) in [(0, 0), (1, 31), (0, 17)]:
            assert np.array_equal(Sh[n, l, h], pv.reconstruct(g, l, h))


# --------------------------------------------------------------------------
# failure detection, checkpoint / resume, write set
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fused", [True, False])
def test_copy_wait_timeout_reports_and_recovers(stepq, fused):
    # every stage expects 16 bytes that never arrive: each block's bounded wait
    # runs out, the error word is set, the pool is untouched, and the context
    # keeps working once the limit is restored
    a = Run(stepq, "qwen_layer", 5)
    b = Run(stepq, "qwen_layer", 5)
    a.pack_initial()
    b.pack_initial()
    a.step(0, fused=fused)
    b.step(0, fused=fused)
    before = a.pool.clone()
    a.ctx.set_wait_limit(4096, 16)
    with pytest.raises(stepq.StepqError) as ei:
        a.step(1, fused=fused)
    assert ei.value.code == stepq.EDEVICE and "copy wait gave up" in str(ei.value)
    assert torch.equal(a.pool, before)
    a.ctx.set_wait_limit(0, 0)
    for t in range(1, 4):
        _, oa = a.step(t, fused=fused)
        _, ob = b.step(t, fused=fused)
        assert np.array_equal(oa, ob)
    assert torch.equal(a.pool, b.pool)


def test_checkpoint_resume_bit_identical(stepq):
    # snapshot the pool to the host mid-run, continue, restore, continue again
    run = Run(stepq, "qwen_pool6", 7, n_layers=2, n_pivots=2)
    run.pack_initial()
    for t in range(3):
        run.step(t, fused=True)
    snap = run.pool.cpu().clone()
    outs = [run.step(t, fused=True)[1] for t in range(3, 6)]
    after = run.pool.clone()
    run.pool.copy_(snap.cuda())
    outs2 = [run.step(t, fused=True)[1] for t in range(3, 6)]
    assert torch.equal(run.pool, after)
    for x, y in zip(outs, outs2):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("fused", [True, False])
def test_write_set_canaries(stepq, fused):
    # the pool sits between canary pages; slots outside the batch stay as they were
    run = Run(stepq, "qwen_pool6", 4, n_layers=2, n_pivots=2, extra_slots=3)
    G = 1 << 16
    buf = torch.full((run.pool.numel() + 2 * G,), 0xA5, dtype=torch.uint8, device="cuda")
    run.pool = buf[G:G + run.pool.numel()]
    run.pool.zero_()
    run.pack_initial()
    idle = [s for s in range(run.n_slots) if s not in set(run.slots.tolist())]
    sb = run.P.slot_bytes
    idle_before = {s: run.pool[s * sb:(s + 1) * sb].clone() for s in idle}
    for t in range(3):
        run.step(t, fused=fused)
    assert bool((buf[:G] == 0xA5).all()) and bool((buf[-G:] == 0xA5).all())
    for s in idle:
        assert torch.equal(run.pool[s * sb:(s + 1) * sb], idle_before[s])


@pytest.mark.parametrize("fused", [True, False])
def test_zero_state_degenerate_fit(stepq, fused):
    # an all-zero state stepped with v = 0: every row takes the 1e-12 floor of r,
    # every column c0 = 1 and a zero least-squares denominator; records must match
    # the oracle bit for bit (FP16 pivot head included) and o must be within the
    # readout tolerance (the kernel's offset-binary bias removal leaves an absolute
    # residual of order 2^-53 sum|k a| (256 + off), about 1e-25 here, where the
    # oracle sums exact zeros)
    run = Run(stepq, "qwen_layer", 3)
    pv = run.pv
    S0 = np.zeros((3, 1, pv.H, pv.D, pv.D), np.float32)
    run.ctx.requant_pack(run.pool, run.slots_t, 3, 0, 1, torch.from_numpy(S0).cuda())
    run.ctx.sync()
    ora = [np.zeros_like(run.slot_bytes_host(n)) for n in range(3)]
    for n in range(3):
        for h in range(pv.H):
            pv.quantize_into(ora[n], 0, h, S0[n, 0, h])
        assert np.array_equal(run.slot_bytes_host(n), ora[n])
    for t in range(3):
        inp = synth.step_inputs(run.wl, run.wl.seed, 3, t, alpha=run.alpha)
        inp["v"] = np.zeros_like(inp["v"])
        d = _inputs_to_dev(inp)
        o = torch.zeros_like(d["q"])
        if fused:
            run.ctx.decode_step_fused(run.pool, run.slots_t, 3, 0, 1, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
        else:
            ws = torch.empty(run.ctx.workspace_bytes(3, 1) // 4, dtype=torch.float32, device="cuda")
            run.ctx.decode_step(run.pool, run.slots_t, 3, 0, 1, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o, ws)
        run.ctx.sync()
        og = o.cpu().numpy()
        assert np.max(np.abs(og)) < 1e-20
        for n in range(3):
            for h in range(pv.H):
                o_ref, tie, S, w = pv.step(ora[n], 0, h, inp["q"][n, 0, h], inp["k"][n, 0, h], inp["v"][n, 0, h],
                                           inp["alpha"][n, 0, h], inp["beta"][n, 0, h])
                assert not np.any(S) and not np.any(o_ref)
                assert _close(og[n, 0, h], o_ref).all()
            assert np.array_equal(run.slot_bytes_host(n), ora[n])
