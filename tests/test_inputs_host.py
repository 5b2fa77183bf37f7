"""Host-side checks of the seeded input generator and the benchmark's
prefill bookkeeping (no GPU: torch on the CPU)."""
import numpy as np
import pytest

from quantized_recurrent_state_b200 import synth

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("name,n,T,lb,le,block", [("tiny_gdn", 2, 7, 0, None, 3), ("gdn_d32", 1, 5, 1, 2, 2),
                                                  ("kda_rows", 1, 3, 4, 6, 256)])
def test_prompt_generator_equals_per_token_draws(name, n, T, lb, le, block):
    """A prompt drawn in blocks of tokens is, token by token, the decode-step
    draw of the same stream (both unit kinds, a layer range, ragged blocks)."""
    wl = synth.workloads()[name]
    alpha = synth.gates(wl, wl.seed)
    P = synth.prompt_inputs_torch(wl, wl.seed, n, 2, T, alpha, "cpu", lb, le, block=block)
    le2 = wl.n_layers if le is None else le
    for t in range(T):
        s = synth.step_inputs_torch(wl, wl.seed, n, 2 + t, alpha, "cpu")
        for k in s:
            assert torch.equal(P[k][:, t], s[k][:, lb:le2]), (t, k)


@pytest.mark.parametrize("name", ["tiny_gdn", "gdn_d32"])
def test_step_inputs_layer_subset_equals_full_draw(name):
    """step_inputs for a subset of layers draws only those blocks of the
    stream: equal to the same layers of the full draw."""
    wl = synth.workloads()[name]
    full = synth.step_inputs(wl, 9, 2, 4)
    layers = list(range(wl.n_layers))[::-1]
    part = synth.step_inputs(wl, 9, 2, 4, layers=layers)
    for k in full:
        assert np.array_equal(part[k], full[k][:, layers]), k


def test_step_inputs_torch_equals_numpy():
    wl = synth.workloads()["gdn_d32"]
    alpha = synth.gates(wl, wl.seed)
    a = synth.step_inputs(wl, wl.seed, 2, 3, alpha=alpha)
    b = synth.step_inputs_torch(wl, wl.seed, 2, 3, alpha, "cpu")
    for k in a:
        assert np.array_equal(a[k], b[k].numpy()), k


def test_prefill_flop_and_byte_counts():
    """The benchmark's algorithmic counts, against their definitions: per
    chunk of c tokens 6 c^2 D + 6 c D^2 + c (c - 1) D FLOPs; per token q, k,
    v, o and the gates, plus the state read and written once."""
    import bench
    D = 128
    assert bench.prefill_flops(64, D) == 6 * 64 * 64 * D + 6 * 64 * D * D + 64 * 63 * D
    assert bench.prefill_flops(100, D) == bench.prefill_flops(64, D) + 6 * 36 * 36 * D + 6 * 36 * D * D + 36 * 35 * D
    assert bench.prefill_flops(0, D) == 0
    assert bench.prefill_bytes(10, D) == 10 * (4 * 4 * D + 8) + 2 * 4 * D * D
    assert bench.prefill_bytes(10, D, rows=True) == 10 * (4 * 4 * D + 4 * D + 4) + 2 * 4 * D * D
