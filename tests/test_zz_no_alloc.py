"""The allocation-free decode step (stepq_decode_step_noalloc).

Some callers cannot allocate device memory: plugins whose host framework owns
every device allocation, or latency-critical serving loops where an
allocator call is not allowed.  For them the library keeps the decode ->
fit-and-pack hand-off values in a fixed array of its own.  This file checks,
through the C ABI, that two consecutive calls of that entry point give the
same readouts and the same packed pool as the
workspace-taking stepq_decode_step (bit for bit, as stepq.h promises), over
a one-layer plan and over a three-layer plan stepped one layer range at a time
with one layer per launch pair (so consecutive calls hand different parts of
the array to different layers while the previous call's fit-and-pack may still
run), and that calls needing more than the array's 8 MiB are refused with a
clear error.  It is collected last so that
a run stopping at the first failure has run every other test first; it also
passes alone in a fresh process.
"""
import numpy as np
import pytest

from quantized_recurrent_state_b200 import synth
from tests._workloads import oracle_plan

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def stepq():
    from quantized_recurrent_state_b200 import build as qbuild
    qbuild.build()
    from quantized_recurrent_state_b200 import stepq as s
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return s


def _setup(stepq, n_req, name="qwen_layer", n_layers=None, n_pivots=None, chunk=4):
    plan, data, wl, _ = oracle_plan(name, n_layers, n_pivots)
    P = stepq.Plan.from_bytes(data)
    ctx = stepq.Context(P, n_req, chunk_layers=chunk)
    slots = torch.arange(n_req, dtype=torch.int32, device="cuda")
    pool = torch.zeros(n_req * P.slot_bytes, dtype=torch.uint8, device="cuda")
    S0 = torch.from_numpy(synth.initial_states(wl, wl.seed, n_req)).cuda()
    ctx.requant_pack(pool, slots, n_req, 0, wl.n_layers, S0)
    ctx.sync()
    return P, wl, ctx, slots, pool


def test_noalloc_matches_workspace_step_two_calls(stepq):
    n = 9
    P, wl, ctx_a, slots, pool_a = _setup(stepq, n)
    _, _, ctx_b, _, pool_b = _setup(stepq, n)
    assert torch.equal(pool_a, pool_b)
    alpha = synth.gates(wl, wl.seed)
    ws = torch.empty(ctx_a.workspace_bytes(n, 1) // 4, dtype=torch.float32, device="cuda")
    for t in range(2):
        d = {k: torch.from_numpy(v).cuda() for k, v in synth.step_inputs(wl, wl.seed, n, t, alpha=alpha).items()}
        o_a = torch.zeros_like(d["q"])
        o_b = torch.zeros_like(d["q"])
        ctx_a.decode_step(pool_a, slots, n, 0, 1, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o_a, ws)
        ctx_a.sync()
        ctx_b.decode_step_noalloc(pool_b, slots, n, 0, 1, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o_b)
        ctx_b.sync()
        assert torch.equal(o_a, o_b), t
        assert torch.equal(pool_a, pool_b), t


def test_noalloc_layer_ranges_one_layer_per_launch(stepq):
    # three layers of the full pool's plan, one layer per launch pair; each step is
    # two calls over [0, 1) and [1, 3) against the same calls of the workspace step
    n = 5
    _, wl, ctx_a, slots, pool_a = _setup(stepq, n, "qwen_pool6", n_layers=3, n_pivots=2, chunk=1)
    _, _, ctx_b, _, pool_b = _setup(stepq, n, "qwen_pool6", n_layers=3, n_pivots=2, chunk=1)
    alpha = synth.gates(wl, wl.seed)
    for t in range(3):
        full = synth.step_inputs(wl, wl.seed, n, t, alpha=alpha)
        for lb, le in ((0, 1), (1, 3)):
            d = {k: torch.from_numpy(np.ascontiguousarray(v[:, lb:le])).cuda() for k, v in full.items()}
            o_a = torch.zeros_like(d["q"])
            o_b = torch.zeros_like(d["q"])
            ws = torch.empty(ctx_a.workspace_bytes(n, le - lb) // 4, dtype=torch.float32, device="cuda")
            ctx_a.decode_step(pool_a, slots, n, lb, le, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o_a, ws)
            ctx_b.decode_step_noalloc(pool_b, slots, n, lb, le, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o_b)
            ctx_a.sync()
            ctx_b.sync()
            assert torch.equal(o_a, o_b), (t, lb)
        assert torch.equal(pool_a, pool_b), t


def test_noalloc_rejects_calls_beyond_its_scratch(stepq):
    n = 2
    P, wl, ctx, slots, pool = _setup(stepq, n)
    big = stepq.NOALLOC_SCRATCH_BYTES // (P.n_heads * P.d * 4) + 1   # requests whose w exceeds the array
    d = {k: torch.from_numpy(v).cuda() for k, v in
         synth.step_inputs(wl, wl.seed, n, 0, alpha=synth.gates(wl, wl.seed)).items()}
    o = torch.zeros_like(d["q"])
    with pytest.raises(stepq.StepqError) as ei:
        ctx.decode_step_noalloc(pool, slots, big, 0, 1, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
    assert ei.value.code == stepq.EINVAL and "scratch" in str(ei.value)
