"""Chunked prefill on the GPU against the token-by-token fp64 recurrence.

The prefill evaluates the gated delta rule in chunks of 64 tokens with the
dense products on the tensor cores (TF32 plus a TF32 remainder) and an fp32
triangular solve (per-head plans: both prefill kernels, the tcgen05 default
and the mma.sync one, run every per-head case), so it matches the oracle to a tolerance, not bit for bit.
Tolerance: each product has relative error about 2^-21 of its terms' sum
(the dropped lo*lo term and the TF32 rounding of the remainders), the fp32
solve about 64 * 2^-24, the gate ratios about |log gamma| 2^-24; over T/64
chunks these add up, and 2e-4 of the largest magnitude (per head) covers
T <= 256 with a wide margin.  Codes written by the packed prefill are
checked bit for bit against the oracle's quantization of the GPU's own fp32
final state.
"""
import numpy as np
import pytest

from oracle import model, prefill
from quantized_recurrent_state_b200 import synth
from tests._workloads import oracle_plan, uniform_plan

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-4


# per-head plans run either prefill kernel; both are checked
KERNELS = ["tcgen05", "mma_sync"]


@pytest.fixture(params=KERNELS)
def pk(request):
    return request.param


def _ctx(stepq, P, n, pk=None):
    ctx = stepq.Context(P, n)
    if pk is not None:
        ctx.set_prefill_kernel(stepq.PREFILL_TCGEN05 if pk == "tcgen05" else stepq.PREFILL_MMA_SYNC)
    return ctx


@pytest.fixture(scope="module")
def stepq():
    from quantized_recurrent_state_b200 import build as qbuild
    qbuild.build()
    from quantized_recurrent_state_b200 import stepq as s
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return s


def _prompt(wl, n, T, seed):
    """[n][T][L][H][D] q, k, v and [n][T][L][H] alpha, beta from the step generator."""
    alpha = synth.gates(wl, seed)
    steps = [synth.step_inputs(wl, seed, n, t, alpha=alpha) for t in range(T)]
    return {key: np.ascontiguousarray(np.stack([s[key] for s in steps], axis=1)) for key in steps[0]}


def _check_head(O_gpu, S_gpu, S0, inp, r, h, l=0):
    O_ref, S_ref = prefill.sequential(S0, inp["q"][r, :, l, h], inp["k"][r, :, l, h], inp["v"][r, :, l, h],
                                      inp["alpha"][r, :, l, h], inp["beta"][r, :, l, h])
    eo = np.max(np.abs(O_gpu - O_ref)) / max(1e-30, np.max(np.abs(O_ref)))
    es = np.max(np.abs(S_gpu - S_ref)) / max(1e-30, np.max(np.abs(S_ref)))
    assert eo <= TOL and es <= TOL, (r, h, eo, es)
    return eo, es


@pytest.mark.parametrize("T", [1, 64, 65, 100, 127, 256])
def test_prefill_fp32_matches_sequential(stepq, pk, T):
    plan, data, wl, _ = oracle_plan("qwen_layer")
    P = stepq.Plan.from_bytes(data)
    n = 2
    ctx = _ctx(stepq, P, n, pk)
    S0 = synth.initial_states(wl, wl.seed, n)                     # [n][1][H][D][D]
    inp = _prompt(wl, n, T, 3000 + T)
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    S = torch.from_numpy(S0).cuda()
    o = torch.zeros_like(d["q"])
    ctx.prefill_fp32(S, n, 0, 1, T, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
    ctx.sync()
    Sg, og = S.cpu().numpy(), o.cpu().numpy()
    worst = (0.0, 0.0)
    for (r, h) in [(0, 0), (1, 7), (0, 23), (1, 47)]:
        e = _check_head(og[r, :, 0, h], Sg[r, 0, h], S0[r, 0, h].astype(np.float64), inp, r, h)
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    print(f"T={T}: worst relative errors o {worst[0]:.2e}, S {worst[1]:.2e}")


def test_prefill_fp32_zero_init_and_empty(stepq, pk):
    plan, data, wl, _ = oracle_plan("qwen_layer")
    P = stepq.Plan.from_bytes(data)
    ctx = _ctx(stepq, P, 1, pk)
    inp = _prompt(wl, 1, 70, 41)
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    S = torch.full((1, 1, wl.n_heads, wl.d, wl.d), float("nan"), dtype=torch.float32, device="cuda")
    o = torch.zeros_like(d["q"])
    ctx.prefill_fp32(S, 1, 0, 1, 70, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o, zero_init=True)
    ctx.sync()
    _check_head(o.cpu().numpy()[0, :, 0, 5], S.cpu().numpy()[0, 0, 5], np.zeros((wl.d, wl.d)), inp, 0, 5)
    before = S.clone()
    ctx.prefill_fp32(S, 1, 0, 1, 0, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)   # T = 0: nothing
    ctx.sync()
    assert torch.equal(S, before)


@pytest.mark.parametrize("from_zero", [False, True])
def test_prefill_into_packed_states(stepq, pk, from_zero):
    plan, data, wl, _ = oracle_plan("qwen_layer")
    pv = model.PlanView(plan)
    P = stepq.Plan.from_bytes(data)
    n, T = 3, 130
    ctx = _ctx(stepq, P, n + 2, pk)
    slots = torch.tensor([4, 0, 2], dtype=torch.int32, device="cuda")
    pool = torch.zeros((n + 2) * P.slot_bytes, dtype=torch.uint8, device="cuda")
    S0 = synth.initial_states(wl, wl.seed, n)
    ctx.requant_pack(pool, slots, n, 0, 1, torch.from_numpy(S0).cuda())
    ctx.sync()
    sb = P.slot_bytes
    before = pool.cpu().numpy().copy()
    inp = _prompt(wl, n, T, 77)
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    o = torch.zeros_like(d["q"])
    ws = torch.empty(ctx.prefill_workspace_bytes(n, 1) // 4, dtype=torch.float32, device="cuda")
    ctx.prefill(pool, slots, n, 0, 1, T, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o, ws, from_zero=from_zero)
    ctx.sync()
    after, og = pool.cpu().numpy(), o.cpu().numpy()
    S_T = ws.view(n, 1, wl.n_heads, wl.d, wl.d).cpu().numpy()   # the last (only) layer's fp32 final states
    slot_of = slots.cpu().numpy()
    for r in range(n):
        s = int(slot_of[r])
        prev_slot = before[s * sb:(s + 1) * sb]
        new_slot = after[s * sb:(s + 1) * sb]
        for h in (0, 9, 30):
            S_start = np.zeros((wl.d, wl.d)) if from_zero else pv.reconstruct(prev_slot, 0, h).astype(np.float64)
            _check_head(og[r, :, 0, h], S_T[r, 0, h], S_start, inp, r, h)
            expect = np.zeros_like(new_slot)
            pv.quantize_into(expect, 0, h, S_T[r, 0, h])
            assert np.array_equal(pv.record(new_slot, 0, h), pv.record(expect, 0, h)), (r, h)
    for s in (1, 3):   # slots outside the batch are untouched
        assert np.array_equal(after[s * sb:(s + 1) * sb], before[s * sb:(s + 1) * sb])


def test_prefill_layer_range_uniform_plan(stepq, pk):
    """Layers [1, 3) of a three-layer uniform 6-bit plan (dual-axis), inputs
    laid out for the range only; layer 0 and slots outside the batch stay put."""
    plan, data, wl, _ = uniform_plan("qwen_pool6", 6, model.QUANT_DUAL_AXIS, n_layers=3)
    pv = model.PlanView(plan)
    P = stepq.Plan.from_bytes(data)
    n, T, lb, le = 2, 70, 1, 3
    ctx = _ctx(stepq, P, 3, pk)
    slots = torch.tensor([2, 0], dtype=torch.int32, device="cuda")
    pool = torch.zeros(3 * P.slot_bytes, dtype=torch.uint8, device="cuda")
    S0 = synth.initial_states(wl, wl.seed, n)
    ctx.requant_pack(pool, slots, n, 0, 3, torch.from_numpy(S0).cuda())
    ctx.sync()
    before = pool.cpu().numpy().copy()
    inp = {k: np.ascontiguousarray(v[:, :, lb:le]) for k, v in _prompt(wl, n, T, 5).items()}
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    o = torch.zeros_like(d["q"])
    ws = torch.empty(ctx.prefill_workspace_bytes(n, le - lb) // 4, dtype=torch.float32, device="cuda")
    assert ctx.prefill_workspace_bytes(n, le - lb) == n * (le - lb) * wl.n_heads * wl.d * wl.d * 4
    ctx.prefill(pool, slots, n, lb, le, T, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o, ws)
    ctx.sync()
    after, og = pool.cpu().numpy(), o.cpu().numpy()
    S_T = ws.view(n, le - lb, wl.n_heads, wl.d, wl.d).cpu().numpy()
    sb = P.slot_bytes
    for r, s in enumerate((2, 0)):
        prev_slot, new_slot = before[s * sb:(s + 1) * sb], after[s * sb:(s + 1) * sb]
        for h in range(wl.n_heads):
            assert np.array_equal(pv.record(new_slot, 0, h), pv.record(prev_slot, 0, h))
        for li, l in enumerate(range(lb, le)):
            for h in (1, 20, 47):
                S_start = pv.reconstruct(prev_slot, l, h).astype(np.float64)
                _check_head(og[r, :, li, h], S_T[r, li, h], S_start, inp, r, h, li)
                expect = np.zeros_like(new_slot)
                pv.quantize_into(expect, l, h, S_T[r, li, h])
                assert np.array_equal(pv.record(new_slot, l, h), pv.record(expect, l, h)), (r, l, h)
    assert np.array_equal(after[sb:2 * sb], before[sb:2 * sb])


def test_prefill_full_pool_sampled(stepq, pk):
    """The launch the prefill benchmark times: a 2,048-token chunk for all
    2,304 heads of the pool (nominal 6 bits, 32 FP16 heads) at batch 1, inputs
    drawn on the device by the same generator.  Sampled heads (and FP16 heads)
    are checked against the token-by-token fp64 recurrence from the records
    the pool held before, and their new records against the oracle's
    quantization of the kernel's final state."""
    plan, data, wl, _ = oracle_plan("qwen_pool6")
    pv = model.PlanView(plan)
    P = stepq.Plan.from_bytes(data)
    n, T, L = 1, 2048, wl.n_layers
    ctx = _ctx(stepq, P, n, pk)
    pool = torch.zeros(n * P.slot_bytes, dtype=torch.uint8, device="cuda")
    slots = torch.arange(n, dtype=torch.int32, device="cuda")
    for l in range(L):
        ctx.requant_pack(pool, slots, n, l, l + 1, synth.initial_states_torch(wl, wl.seed, n, l, "cuda"))
    inp = synth.prompt_inputs_torch(wl, wl.seed, n, 0, T, synth.gates(wl, wl.seed), "cuda")
    o = torch.zeros_like(inp["q"])
    ws = torch.empty(ctx.prefill_workspace_bytes(n, L) // 4, dtype=torch.float32, device="cuda")
    ctx.sync()
    before = pool.cpu().numpy().copy()
    ctx.prefill(pool, slots, n, 0, L, T, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, ws)
    ctx.sync()
    after = pool.cpu().numpy()
    S_T = ws.view(n, L, wl.n_heads, wl.d, wl.d)
    rng = np.random.default_rng(21)
    units = P.widths().reshape(L * wl.n_heads, -1)
    piv = np.nonzero((units == 16).any(axis=1))[0]
    samples = [(int(rng.integers(L)), int(rng.integers(wl.n_heads))) for _ in range(6)]
    samples += [(int(u) // wl.n_heads, int(u) % wl.n_heads) for u in piv[:2]]
    worst = (0.0, 0.0)
    for (l, h) in samples:
        x = {k: v[:, :, l:l + 1, h:h + 1].cpu().numpy() for k, v in inp.items()}
        S_start = pv.reconstruct(before, l, h).astype(np.float64)
        s_t = S_T[0, l, h].cpu().numpy()
        e = _check_head(o[0, :, l, h].cpu().numpy(), s_t, S_start, x, 0, 0, 0)
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        expect = np.zeros_like(after)
        pv.quantize_into(expect, l, h, s_t)
        assert np.array_equal(pv.record(after, l, h), pv.record(expect, l, h)), (l, h)
    print(f"full pool, T={T}: worst relative errors o {worst[0]:.2e}, S {worst[1]:.2e}")


def _check_record(pv, new_slot, l, h, S):
    """The record the GPU wrote for (l, h) against the oracle's quantization of
    the kernel's fp32 state S: bit-exact except codes the oracle marks as ties."""
    expect = np.zeros_like(new_slot)
    tie = pv.quantize_into(expect, l, h, S)
    rg, ro = pv.record(new_slot, l, h), pv.record(expect, l, h)
    if np.array_equal(rg, ro):
        return
    zg, hg, _, _ = model.unpack_head(pv.mode, pv.D, pv.rw(l, h), rg)
    zo, ho, _, _ = model.unpack_head(pv.mode, pv.D, pv.rw(l, h), ro)
    assert not (((zg != zo) | (hg != ho)) & (tie == 0)).any(), (l, h)


# ---- per-key-row gates (KDA units) -----------------------------------------

@pytest.mark.parametrize("T", [1, 64, 100, 256])
def test_prefill_rows_fp32_matches_sequential(stepq, T):
    plan, data, wl, _ = oracle_plan("kda_rows", n_layers=1, n_pivots=8)
    P = stepq.Plan.from_bytes(data)
    n = 2
    ctx = stepq.Context(P, n)
    S0 = synth.initial_states(wl, wl.seed, n)
    inp = _prompt(wl, n, T, 4000 + T)
    assert inp["alpha"].shape == (n, T, 1, wl.n_heads, wl.d)
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    S = torch.from_numpy(S0).cuda()
    o = torch.zeros_like(d["q"])
    ctx.prefill_fp32(S, n, 0, 1, T, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
    ctx.sync()
    Sg, og = S.cpu().numpy(), o.cpu().numpy()
    worst = (0.0, 0.0)
    for (r, h) in [(0, 0), (1, 7), (0, 19), (1, 31)]:
        e = _check_head(og[r, :, 0, h], Sg[r, 0, h], S0[r, 0, h].astype(np.float64), inp, r, h)
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    print(f"rows T={T}: worst relative errors o {worst[0]:.2e}, S {worst[1]:.2e}")


@pytest.mark.parametrize("from_zero", [False, True])
def test_prefill_rows_into_packed_states(stepq, from_zero):
    """Layers [1, 3) of a three-layer per-row plan (pivot rows included)."""
    plan, data, wl, _ = oracle_plan("kda_rows", n_layers=3, n_pivots=24)
    pv = model.PlanView(plan)
    P = stepq.Plan.from_bytes(data)
    n, T, lb, le = 2, 130, 1, 3
    ctx = stepq.Context(P, 3)
    slots = torch.tensor([2, 0], dtype=torch.int32, device="cuda")
    pool = torch.zeros(3 * P.slot_bytes, dtype=torch.uint8, device="cuda")
    ctx.requant_pack(pool, slots, n, 0, 3, torch.from_numpy(synth.initial_states(wl, wl.seed, n)).cuda())
    ctx.sync()
    before = pool.cpu().numpy().copy()
    inp = {k: np.ascontiguousarray(v[:, :, lb:le]) for k, v in _prompt(wl, n, T, 6).items()}
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    o = torch.zeros_like(d["q"])
    ws = torch.empty(ctx.prefill_workspace_bytes(n, le - lb) // 4, dtype=torch.float32, device="cuda")
    ctx.prefill(pool, slots, n, lb, le, T, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o, ws, from_zero=from_zero)
    ctx.sync()
    after, og = pool.cpu().numpy(), o.cpu().numpy()
    S_T = ws.view(n, le - lb, wl.n_heads, wl.d, wl.d).cpu().numpy()
    sb = P.slot_bytes
    units = P.widths().reshape(3, wl.n_heads, -1)
    for r, s in enumerate((2, 0)):
        prev_slot, new_slot = before[s * sb:(s + 1) * sb], after[s * sb:(s + 1) * sb]
        assert np.array_equal(new_slot[:int(pv.offsets[wl.n_heads])], prev_slot[:int(pv.offsets[wl.n_heads])])
        for li, l in enumerate(range(lb, le)):
            heads = [0, 13, 31] + [int(x) for x in np.nonzero((units[l] == 16).any(axis=1))[0][:2]]
            for h in heads:
                S_start = np.zeros((wl.d, wl.d)) if from_zero else pv.reconstruct(prev_slot, l, h).astype(np.float64)
                _check_head(og[r, :, li, h], S_T[r, li, h], S_start, inp, r, h, li)
                _check_record(pv, new_slot, l, h, S_T[r, li, h])
    assert np.array_equal(after[sb:2 * sb], before[sb:2 * sb])


def test_prefill_degenerate_gates_full_pool(stepq, pk):
    """alpha = 1, beta = 0 for every token of the whole pool (2,304 heads, batch
    1, 300 tokens): M = 0 and the update adds exact zeros, so the fp32 state
    comes back bit for bit, and o_t = S_0^T q_t."""
    plan, data, wl, _ = uniform_plan("qwen_pool6", 6, model.QUANT_DUAL_AXIS)
    P = stepq.Plan.from_bytes(data)
    n, T, L = 1, 300, wl.n_layers
    ctx = _ctx(stepq, P, n, pk)
    inp = synth.prompt_inputs_torch(wl, wl.seed, n, 0, T, synth.gates(wl, wl.seed), "cuda")
    inp["alpha"].fill_(1.0)
    inp["beta"].zero_()
    S0 = torch.cat([synth.initial_states_torch(wl, wl.seed, n, l, "cuda") for l in range(L)], dim=1)
    S = S0.clone()
    o = torch.zeros_like(inp["q"])
    ctx.prefill_fp32(S, n, 0, L, T, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o)
    ctx.sync()
    assert torch.equal(S, S0)
    ref = torch.einsum("nlhij,ntlhi->ntlhj", S0.double(), inp["q"].double())
    err = (o.double() - ref).abs().amax(dim=(1, 4)) / ref.abs().amax(dim=(1, 4))
    assert float(err.max()) <= TOL, float(err.max())


def test_packed_prefill_noop_calls(stepq, pk):
    """T = 0 and n_req = 0 leave the pool as it was."""
    plan, data, wl, _ = oracle_plan("qwen_layer")
    P = stepq.Plan.from_bytes(data)
    ctx = _ctx(stepq, P, 2, pk)
    slots = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    pool = torch.zeros(2 * P.slot_bytes, dtype=torch.uint8, device="cuda")
    ctx.requant_pack(pool, slots, 2, 0, 1, torch.from_numpy(synth.initial_states(wl, wl.seed, 2)).cuda())
    ctx.sync()
    before = pool.clone()
    inp = {k: torch.from_numpy(v).cuda() for k, v in _prompt(wl, 2, 3, 8).items()}
    o = torch.zeros_like(inp["q"])
    ws = torch.empty(ctx.prefill_workspace_bytes(2, 1) // 4, dtype=torch.float32, device="cuda")
    ctx.prefill(pool, slots, 2, 0, 1, 0, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, ws)
    ctx.prefill(pool, slots, 0, 0, 1, 3, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, ws)
    ctx.sync()
    assert torch.equal(pool, before)


def test_prefill_gates_out_of_range_are_reported(stepq):
    """Per-row gates whose 32-token log-products leave the fp32 range, and a
    per-head gate of 0, set the device error word (stepq_sync fails with
    "prefill gate out of range"); the next valid call runs clean."""
    plan, data, wl, _ = oracle_plan("kda_rows", n_layers=1, n_pivots=8)
    ctx = stepq.Context(stepq.Plan.from_bytes(data), 1)
    inp = {k: torch.from_numpy(v).cuda() for k, v in _prompt(wl, 1, 64, 12).items()}
    S = torch.zeros((1, 1, wl.n_heads, wl.d, wl.d), dtype=torch.float32, device="cuda")
    o = torch.zeros_like(inp["q"])
    bad = inp["alpha"].clone()
    bad[0, :, 0, 3, 17] = 1e-3                      # one key row: 32 * ln(1e-3) = -221
    ctx.prefill_fp32(S, 1, 0, 1, 64, inp["q"], inp["k"], inp["v"], bad, inp["beta"], o, zero_init=True)
    with pytest.raises(stepq.StepqError, match="prefill gate out of range"):
        ctx.sync()
    ctx.prefill_fp32(S, 1, 0, 1, 64, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, zero_init=True)
    ctx.sync()
    _check_head(o.cpu().numpy()[0, :, 0, 3], S.cpu().numpy()[0, 0, 3], np.zeros((wl.d, wl.d)),
                {k: v.cpu().numpy() for k, v in inp.items()}, 0, 3)

    plan, data, wl, _ = oracle_plan("qwen_layer")
    ctx = stepq.Context(stepq.Plan.from_bytes(data), 1)     # per-head plans: the default (tcgen05) kernel
    inp = {k: torch.from_numpy(v).cuda() for k, v in _prompt(wl, 1, 10, 13).items()}
    S = torch.zeros((1, 1, wl.n_heads, wl.d, wl.d), dtype=torch.float32, device="cuda")
    o = torch.zeros_like(inp["q"])
    bad = inp["alpha"].clone()
    bad[0, 4, 0, 7] = 0.0
    ctx.prefill_fp32(S, 1, 0, 1, 10, inp["q"], inp["k"], inp["v"], bad, inp["beta"], o, zero_init=True)
    with pytest.raises(stepq.StepqError, match="prefill gate out of range"):
        ctx.sync()
    ctx.prefill_fp32(S, 1, 0, 1, 10, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, zero_init=True)
    ctx.sync()


@pytest.mark.parametrize("name,kern", [("qwen_layer", "tcgen05"), ("qwen_layer", "mma_sync"), ("kda_rows", None)])
def test_prefill_then_decode(stepq, name, kern):
    """The serving order: a 100-token prompt prefilled into packed states,
    then 3 fused decode steps from the records the prefill wrote, checked
    against the oracle stepping the same records (codes bit-exact up to
    rounding ties, o within rtol 1e-4 / atol 1e-5)."""
    kw = {"n_layers": 1, "n_pivots": 8} if name == "kda_rows" else {}
    plan, data, wl, _ = oracle_plan(name, **kw)
    pv = model.PlanView(plan)
    P = stepq.Plan.from_bytes(data)
    n, T = 2, 100
    ctx = _ctx(stepq, P, n, kern)
    slots = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    pool = torch.zeros(n * P.slot_bytes, dtype=torch.uint8, device="cuda")
    ctx.requant_pack(pool, slots, n, 0, 1, torch.from_numpy(synth.initial_states(wl, wl.seed, n)).cuda())
    inp = {k: torch.from_numpy(v).cuda() for k, v in _prompt(wl, n, T, 31).items()}
    o = torch.zeros_like(inp["q"])
    ws = torch.empty(ctx.prefill_workspace_bytes(n, 1) // 4, dtype=torch.float32, device="cuda")
    ctx.prefill(pool, slots, n, 0, 1, T, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, ws)
    ctx.sync()
    ref = pool.cpu().numpy().copy()          # the oracle continues from the records the prefill wrote
    sb = P.slot_bytes
    alpha = synth.gates(wl, wl.seed)
    slot_of = slots.cpu().numpy()
    od = torch.zeros((n, 1, wl.n_heads, wl.d), dtype=torch.float32, device="cuda")
    for t in range(3):
        x = synth.step_inputs(wl, wl.seed + 1, n, T + t, alpha=alpha)
        d = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in x.items()}
        ctx.decode_step_fused(pool, slots, n, 0, 1, d["q"], d["k"], d["v"], d["alpha"], d["beta"], od)
        ctx.sync()
        got, og = pool.cpu().numpy(), od.cpu().numpy()
        for r in range(n):
            s = int(slot_of[r])
            slot = ref[s * sb:(s + 1) * sb]
            for h in range(wl.n_heads):
                o_ref, tie, S, w = pv.step(slot, 0, h, x["q"][r, 0, h], x["k"][r, 0, h], x["v"][r, 0, h],
                                           x["alpha"][r, 0, h], x["beta"][r, 0, h])
                assert (np.abs(og[r, 0, h] - o_ref) <= 1e-5 + 1e-4 * np.abs(o_ref)).all(), (t, r, h)
                rg, ro = pv.record(got[s * sb:(s + 1) * sb], 0, h), pv.record(slot, 0, h)
                if not np.array_equal(rg, ro):
                    zg, hg, _, _ = model.unpack_head(pv.mode, pv.D, pv.rw(0, h), rg)
                    zo, ho, _, _ = model.unpack_head(pv.mode, pv.D, pv.rw(0, h), ro)
                    assert not (((zg != zo) | (hg != ho)) & (tie == 0)).any(), (t, r, h)
            ref[s * sb:(s + 1) * sb] = slot
        # continue both from the oracle's records, so a tie never compounds
        pool.copy_(torch.from_numpy(ref).cuda())


# ---- the tensor-memory (tcgen05) prefill kernel for per-head plans ------------------

@pytest.mark.parametrize("T", [1, 65, 200])
def test_prefill_tcgen05_matches_sequential(stepq, T):
    plan, data, wl, _ = oracle_plan("qwen_layer")
    ctx = stepq.Context(stepq.Plan.from_bytes(data), 2)
    ctx.set_prefill_kernel(stepq.PREFILL_TCGEN05)
    S0 = synth.initial_states(wl, wl.seed, 2)
    inp = _prompt(wl, 2, T, 5000 + T)
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    S = torch.from_numpy(S0).cuda()
    o = torch.zeros_like(d["q"])
    ctx.prefill_fp32(S, 2, 0, 1, T, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
    ctx.sync()
    Sg, og = S.cpu().numpy(), o.cpu().numpy()
    for (r, h) in [(0, 0), (1, 11), (0, 30), (1, 47)]:
        _check_head(og[r, :, 0, h], Sg[r, 0, h], S0[r, 0, h].astype(np.float64), inp, r, h)


def test_prefill_tcgen05_packed_layer_range_and_gate_errors(stepq):
    plan, data, wl, _ = uniform_plan("qwen_pool6", 6, model.QUANT_DUAL_AXIS, n_layers=3)
    pv = model.PlanView(plan)
    P = stepq.Plan.from_bytes(data)
    n, T, lb, le = 2, 130, 1, 3
    ctx = stepq.Context(P, 2)
    ctx.set_prefill_kernel(stepq.PREFILL_TCGEN05)
    slots = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    pool = torch.zeros(2 * P.slot_bytes, dtype=torch.uint8, device="cuda")
    ctx.requant_pack(pool, slots, n, 0, 3, torch.from_numpy(synth.initial_states(wl, wl.seed, n)).cuda())
    ctx.sync()
    before = pool.cpu().numpy().copy()
    inp = {k: np.ascontiguousarray(v[:, :, lb:le]) for k, v in _prompt(wl, n, T, 9).items()}
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    o = torch.zeros_like(d["q"])
    ws = torch.empty(ctx.prefill_workspace_bytes(n, le - lb) // 4, dtype=torch.float32, device="cuda")
    ctx.prefill(pool, slots, n, lb, le, T, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o, ws)
    ctx.sync()
    after, og = pool.cpu().numpy(), o.cpu().numpy()
    S_T = ws.view(n, le - lb, wl.n_heads, wl.d, wl.d).cpu().numpy()
    sb = P.slot_bytes
    for r, s in enumerate((1, 0)):
        prev_slot, new_slot = before[s * sb:(s + 1) * sb], after[s * sb:(s + 1) * sb]
        for li, l in enumerate(range(lb, le)):
            for h in (0, 25, 47):
                _check_head(og[r, :, li, h], S_T[r, li, h], pv.reconstruct(prev_slot, l, h).astype(np.float64),
                            inp, r, h, li)
                _check_record(pv, new_slot, l, h, S_T[r, li, h])
    bad = d["alpha"].clone()
    bad[0, 3, 0, 5] = 0.0
    ctx.prefill(pool, slots, n, lb, le, T, d["q"], d["k"], d["v"], bad, d["beta"], o, ws)
    with pytest.raises(stepq.StepqError, match="prefill gate out of range"):
        ctx.sync()


def test_prefill_tcgen05_setting_leaves_per_row_plans_on_mma_sync(stepq):
    plan, data, wl, _ = oracle_plan("kda_rows", n_layers=1, n_pivots=8)
    ctx = stepq.Context(stepq.Plan.from_bytes(data), 1)
    ctx.set_prefill_kernel(stepq.PREFILL_TCGEN05)
    with pytest.raises(stepq.StepqError):
        ctx.set_prefill_kernel(7)
    S0 = synth.initial_states(wl, wl.seed, 1)
    inp = _prompt(wl, 1, 70, 4)
    d = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    S = torch.from_numpy(S0).cuda()
    o = torch.zeros_like(d["q"])
    ctx.prefill_fp32(S, 1, 0, 1, 70, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
    ctx.sync()
    _check_head(o.cpu().numpy()[0, :, 0, 9], S.cpu().numpy()[0, 0, 9], S0[0, 0, 9].astype(np.float64), inp, 0, 9)
