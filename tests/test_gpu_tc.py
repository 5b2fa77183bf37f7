"""The tensor-core (tcgen05, TF32) building blocks against fp64 products of
the TF32-truncated operands: a product with both operands in shared memory, a
product whose A is the accumulator the first one left in tensor memory, and
one whose A was written to tensor memory."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _tf32(x: np.ndarray) -> np.ndarray:
    """fp32 values with the low 13 mantissa bits dropped, as fp64."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return b.view(np.float32).astype(np.float64)


def test_tcgen05_tf32_products():
    from quantized_recurrent_state_b200 import build as qbuild
    qbuild.build()
    from quantized_recurrent_state_b200 import stepq
    g = np.random.default_rng(17)
    A = g.standard_normal((128, 32)).astype(np.float32)
    B1 = g.standard_normal((32, 32)).astype(np.float32)
    B2 = g.standard_normal((64, 32)).astype(np.float32)
    dA, dB1, dB2 = (torch.from_numpy(x).cuda() for x in (A, B1, B2))
    D1 = torch.full((128, 32), float("nan"), device="cuda")
    D2 = torch.full((128, 64), float("nan"), device="cuda")
    D3 = torch.full((128, 64), float("nan"), device="cuda")
    stepq.selftest_tc(dA, dB1, dB2, D1, D2, D3)
    d1, d2, d3 = (x.cpu().numpy() for x in (D1, D2, D3))
    for got, ref in ((d1, _tf32(A) @ _tf32(B1).T), (d2, _tf32(d1) @ _tf32(B2).T), (d3, _tf32(A) @ _tf32(B2).T)):
        # fp32 accumulation of 32 exact products
        assert np.abs(got - ref).max() <= 1e-6 * np.abs(ref).max(), np.abs(got - ref).max() / np.abs(ref).max()
