"""Long-horizon drift study (short run): packed path vs FP32-state kernel.

On the drift workload every half-life is 1,000-20,000 steps, so the
quantization error written back each step barely decays (背景与动机).  The
test checks that the recorded error follows E_t = A_t E_{t-1} + eps_t to
fp32 rounding, that the errors are finite, and that they order with the
bit budget (uniform INT8 < nominal 6-bit < nominal 4-bit; absmax INT8 <
absmax INT6 < absmax INT4).
"""
import math

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_drift_short():
    from quantized_recurrent_state_b200 import drift
    out = drift.run(steps=512, every=128, checks=2)
    print(out)
    for kind, r in out["plans"].items():
        assert math.isfinite(r["readout_rel_err_max"]), kind
        for _, e in r["state_rel_err"]:
            assert math.isfinite(e) and e < 2.0, kind
        for _, res in r["error_recursion_residual"]:
            assert res < 1e-4, (kind, res)
    p = out["plans"]
    assert p["int8"]["readout_rel_err_mean"] < p["nominal6"]["readout_rel_err_mean"] < p["nominal4"]["readout_rel_err_mean"]
    assert (p["absmax8"]["readout_rel_err_mean"] < p["absmax6"]["readout_rel_err_mean"]
            < p["absmax4"]["readout_rel_err_mean"])
