"""The plan the benchmark times, built on the GPU, against the oracle's plan.

The benchmark calibrates on the device (FP32-state recurrence, the row-impact
and distortion kernels) and builds the plan with the library's planner.  The
oracle calibrates the same seeded inputs on the CPU and allocates with its own
DP / Lagrangian.  Unit widths and pivot placement must agree bit for bit
(paper digest page, 方法-1: the offline precision map; 方法-2: row impact).
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


@pytest.mark.parametrize("name", ["qwen_pool6", "qwen_pool4", "kda_rows"])
def test_benchmark_plan_equals_oracle_plan(stepq, name):
    import bench
    wl = synth.workloads()[name]
    P, _ = bench.product_plan(stepq, synth, wl, "cuda")
    plan, _, _, stats = oracle_plan(name)
    w_gpu = np.asarray(P.widths(), np.int64)
    w_ora = np.asarray(plan["widths"], np.int64)
    assert w_gpu.shape == w_ora.shape
    piv_gpu = np.nonzero(w_gpu == 16)[0]
    piv_ora = np.nonzero(w_ora == 16)[0]
    assert np.array_equal(piv_gpu, piv_ora), (name, piv_gpu[:8], piv_ora[:8])
    diff = np.nonzero(w_gpu != w_ora)[0]
    assert diff.size == 0, (name, diff.size, diff[:8])
    info = P.info
    assert info.n_pivots == wl.n_pivots
    print(f"{name}: {w_gpu.size} units, {piv_gpu.size} pivots, widths identical; "
          f"bits/value {info.bits_per_value:.4f} ({info.bits_per_value_s16:.4f} with 16-bit scales)")
