"""Host-side checks of libstepq.so that need no GPU: the library loads, exports
every entry point its header declares, parses and validates plan files
written by the oracle's independent writer, and its offline planner picks
the same widths and pivots as the oracle's allocator on the same statistics.
"""
import os
import re
import struct
import zlib

import numpy as np
import pytest

from oracle import allocator, model, plan_io
from quantized_recurrent_state_b200 import build as qbuild
from quantized_recurrent_state_b200 import stepq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    qbuild.build()


def test_exports_every_declared_symbol():
    hdr = open(os.path.join(ROOT, "include", "stepq.h")).read()
    declared = set(re.findall(r"^\s*(?:const char \*|int|void|size_t|uint64_t)\s*\*?\s*(stepq_\w+)\s*\(", hdr, re.M))
    assert len(declared) >= 20
    l = stepq.lib()
    for name in declared:
        assert hasattr(l, name), name
    assert declared == set(stepq.EXPORTED)


def _tiny_plan_dict(mode=0):
    D = 16
    if mode == 0:
        widths = np.array([2, 6, 16, 4], np.uint8)
        units = 4
    else:
        rng = np.random.default_rng(3)
        widths = rng.choice([4, 6, 8], size=4 * D).astype(np.uint8)
        widths[[3, 40]] = 16
        # keep inside the budget
        while widths[widths != 16].astype(int).sum() > 6 * (widths != 16).sum():
            widths[np.argmax(widths * (widths != 16))] -= 2
        units = 4 * D
    return dict(mode=mode, n_layers=2, n_heads=2, d=D, n_pivots=int((widths == 16).sum()),
                bitset=[2, 4, 6] if mode == 0 else [4, 6, 8], nominal_bits=4.0 if mode == 0 else 6.0,
                horizon=65536, widths=widths, wbar=np.linspace(0.5, 2.0, 4 * D).astype(np.float32),
                rho=np.linspace(0.8, 1.2, 4 * D).astype(np.float32), lgate=-np.linspace(0.01, 0.1, units),
                lifetime=np.linspace(1, 10, units))


@pytest.mark.parametrize("mode", [0, 1])
def test_plan_parse_matches_oracle_layout(mode):
    pd = _tiny_plan_dict(mode)
    data = plan_io.write_plan(None, pd)
    p = stepq.Plan.from_bytes(data)
    assert (p.mode, p.n_layers, p.n_heads, p.d) == (mode, 2, 2, 16)
    assert np.array_equal(p.widths(), pd["widths"])
    offs, slot = plan_io.pool_layout(pd)
    assert p.slot_bytes == slot
    for l in range(2):
        for h in range(2):
            off, nb = p.record(l, h)
            assert off == offs[l * 2 + h]
            assert nb == plan_io.record_bytes(mode, 16, plan_io.head_row_widths(pd, l, h))
    assert p.info.bits_per_value == pytest.approx(allocator.bits_per_value(mode, 2, 2, 16, pd["widths"]), rel=1e-15)
    assert p.info.bits_per_value_s16 == pytest.approx(
        allocator.bits_per_value(mode, 2, 2, 16, pd["widths"], scale_bits=16), rel=1e-15)
    assert p.info.n_pivots == pd["n_pivots"]


def _expect_format_error(data):
    with pytest.raises(stepq.StepqError) as ei:
        stepq.Plan.from_bytes(data)
    assert ei.value.code == stepq.EFORMAT, str(ei.value)


def _recrc(b: bytearray) -> bytes:
    b[-4:] = struct.pack("<I", zlib.crc32(bytes(b[:-4])) & 0xFFFFFFFF)
    return bytes(b)


def test_plan_validation_errors():
    pd = _tiny_plan_dict(0)
    good = bytearray(plan_io.write_plan(None, pd))
    bad = bytearray(good); bad[0] = ord("X"); _expect_format_error(_recrc(bad))                 # magic
    bad = bytearray(good); bad[70] ^= 1; _expect_format_error(bytes(bad))                        # CRC
    bad = bytearray(good); bad[8] = 2; _expect_format_error(_recrc(bad))                         # version
    _expect_format_error(bytes(good[:-8]))                                                       # truncated
    bad = bytearray(good); bad[36] = 2; _expect_format_error(_recrc(bad))                        # pivot count
    bad = bytearray(good); bad[64 + 0] = 8; _expect_format_error(_recrc(bad))                    # width not in bitset
    pd2 = dict(pd); pd2["widths"] = np.array([6, 6, 16, 4], np.uint8)                            # 16 bits > floor(4*3)
    _expect_format_error(plan_io.write_plan(None, pd2))
    pd3 = dict(pd); pd3["wbar"] = pd["wbar"].copy(); pd3["wbar"][5] = 0.0                       # non-positive weight
    _expect_format_error(plan_io.write_plan(None, pd3))
    with pytest.raises(stepq.StepqError) as ei:
        stepq.Plan.load("/nonexistent/plan.bin")
    assert ei.value.code == stepq.EINVAL


def _random_stats(mode, L, H, D, bits, seed):
    rng = np.random.default_rng(seed)
    units = L * H if mode == 0 else L * H * D
    lgate = -np.log(2) / np.exp(rng.uniform(np.log(4), np.log(20000), units))
    # decreasing distortion in the width
    base = rng.uniform(0.5, 2.0, units)[:, None]
    rate = rng.uniform(0.4, 0.8, units)[:, None]
    dist = base * np.exp(-rate * np.asarray(bits, float)[None, :])
    wbar = rng.uniform(0.2, 5.0, L * H * D).astype(np.float32)
    return dict(lgate=lgate, dist=dist, wbar=wbar,
                rho=(1.0 / np.sqrt(np.sqrt(wbar.astype(np.float64)))).astype(np.float32))


@pytest.mark.parametrize("mode,bits,nominal,pivots", [(0, (4, 6, 8), 6.0, 5), (0, (2, 4, 6, 8), 4.0, 3),
                                                       (1, (4, 6, 8), 6.0, 40), (1, (2, 4, 6, 8), 4.0, 7)])
def test_product_planner_equals_oracle_allocator(mode, bits, nominal, pivots):
    L, H, D = 3, 8, 16
    for seed in range(3):
        st = _random_stats(mode, L, H, D, bits, seed)
        ora = model.build_plan(mode, D, L, H, st, bits, nominal, pivots, 65536)
        p = stepq.Plan.build(mode, L, H, D, bits, nominal, pivots, 65536, st["lgate"], st["dist"], st["wbar"])
        assert np.array_equal(p.widths(), ora["widths"]), (mode, seed)
        # rho derived identically
        data = plan_io.write_plan(None, ora)
        assert plan_io.read_plan(data)["rho"].tobytes() == ora["rho"].tobytes()


def test_product_planner_writes_file(tmp_path):
    st = _random_stats(0, 2, 4, 16, (4, 6, 8), 9)
    path = str(tmp_path / "p.plan")
    p = stepq.Plan.build(0, 2, 4, 16, (4, 6, 8), 6.0, 1, 4096, st["lgate"], st["dist"], st["wbar"], path=path)
    back = plan_io.read_plan(open(path, "rb").read())
    assert np.array_equal(back["widths"], p.widths())
    assert np.array_equal(back["rho"], st["rho"])


def test_calls_without_device_fail_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    pd = _tiny_plan_dict(0)
    p = stepq.Plan.from_bytes(plan_io.write_plan(None, pd))
    import ctypes
    h = ctypes.c_void_p()
    rc = stepq.lib().stepq_ctx_create(p._h, ctypes.c_void_p(1), ctypes.c_void_p(2), 4, 1, ctypes.byref(h))
    assert rc == stepq.ECUDA


@pytest.mark.parametrize("sbits", [32, 16])
@pytest.mark.parametrize("mode,quant", [(0, stepq.QUANT_ABSMAX), (0, stepq.QUANT_DUAL_AXIS), (1, stepq.QUANT_DUAL_AXIS)])
def test_uniform_plan_file_matches_oracle(tmp_path, mode, quant, sbits):
    L, H, D = 2, 3, 16
    wbar = np.linspace(0.5, 2.0, L * H * D).astype(np.float32)
    path = str(tmp_path / "u.plan")
    p = stepq.Plan.build_uniform(mode, L, H, D, 6, quant, 4096, wbar, path=path, scale_bits=sbits)
    ora = model.uniform_plan(mode, D, L, H, 6, quant, 4096, wbar, scale_bits=sbits)
    assert open(path, "rb").read() == plan_io.write_plan(None, ora)
    assert p.info.quantizer == quant and p.info.n_pivots == 0 and p.info.scale_bits == sbits
    assert p.info.bits_per_value == pytest.approx(
        allocator.bits_per_value(mode, L, H, D, ora["widths"], scale_bits=sbits), rel=1e-15)
    offs, slot = plan_io.pool_layout(ora)
    assert p.slot_bytes == slot
    for l in range(L):
        for h in range(H):
            assert p.record(l, h)[0] == offs[l * H + h]
    assert p.info.units_by_width[6] == p.info.n_units


def test_quantizer_field_validation():
    good = bytearray(plan_io.write_plan(None, model.uniform_plan(0, 16, 2, 2, 4, model.QUANT_ABSMAX, 4096)))
    assert stepq.Plan.from_bytes(bytes(good)).info.quantizer == stepq.QUANT_ABSMAX
    bad = bytearray(good); bad[56] = 2; _expect_format_error(_recrc(bad))                        # unknown quantizer
    bad = bytearray(good); bad[60] = 1; _expect_format_error(_recrc(bad))                        # scale word
    ok16 = bytearray(good); ok16[60] = 16
    assert stepq.Plan.from_bytes(_recrc(ok16)).info.scale_bits == 16
    kda = bytearray(plan_io.write_plan(None, model.uniform_plan(1, 16, 2, 2, 4, 0, 4096)))
    kda[56] = 1; _expect_format_error(_recrc(kda))                                               # absmax needs mode 0
    with pytest.raises(stepq.StepqError) as ei:
        stepq.Plan.build_uniform(1, 2, 2, 16, 4, stepq.QUANT_ABSMAX)
    assert ei.value.code == stepq.EINVAL


@pytest.mark.parametrize("mode,sbits", [(0, 32), (0, 16), (1, 32)])
def test_plan_slice_matches_oracle(mode, sbits):
    L, H, D = 5, 4, 16
    bits = (4, 6, 8)
    st = _random_stats(mode, L, H, D, bits, 21)
    pivots = 3 if mode == 0 else 12
    ora = model.build_plan(mode, D, L, H, st, bits, 6.0, pivots, 4096, scale_bits=sbits)
    p = stepq.Plan.from_bytes(plan_io.write_plan(None, ora))
    for lb, le in ((0, 5), (1, 3), (4, 5), (0, 1)):
        sp = p.slice(lb, le)
        so = model.slice_plan(ora, lb, le)
        assert (sp.n_layers, sp.info.n_pivots, sp.info.scale_bits) == (le - lb, so["n_pivots"], sbits)
        assert np.array_equal(sp.widths(), so["widths"])
        assert sp.info.nominal_bits == np.float32(so["nominal_bits"])
        # the oracle's own file of the slice parses to the same plan
        back = stepq.Plan.from_bytes(plan_io.write_plan(None, so))
        assert back.slot_bytes == sp.slot_bytes
        offs, slot = plan_io.pool_layout(so)
        assert sp.slot_bytes == slot
        for l in range(le - lb):
            for h in range(H):
                assert sp.record(l, h) == (int(offs[l * H + h]), plan_io.record_bytes(
                    mode, D, plan_io.head_row_widths(so, l, h), sbits))
    with pytest.raises(stepq.StepqError):
        p.slice(3, 3)


def test_new_entry_points_reject_bad_arguments_without_a_device():
    """Argument checks come before any CUDA call: a null context or pointer, or an
    unknown prefill kernel, is STEPQ_EINVAL with a message."""
    l = stepq.lib()
    assert l.stepq_ctx_set_prefill_kernel(None, stepq.PREFILL_TCGEN05) == stepq.EINVAL
    assert b"null context" in l.stepq_last_error()
    assert l.stepq_ctx_set_step_kernel(None, stepq.STEP_TMEM) == stepq.EINVAL
    assert b"null context" in l.stepq_last_error()
    assert l.stepq_selftest_tc(None, None, None, None, None, None) == stepq.EINVAL
    assert b"A" in l.stepq_last_error()
    assert l.stepq_prefill_workspace_bytes(None, 1, 1) == 0


@pytest.mark.parametrize("scale_bits", [32, 16])
@pytest.mark.parametrize("bits", [2, 4, 6, 8])
def test_benchmark_byte_model_per_head_step(bits, scale_bits):
    """The roofline's algorithmic bytes, from the library's own record sizes,
    against the closed form of one per-head-unit step at d = 128: the record
    (D^2 b / 8 code bytes + r and c, 4 or 2 bytes each per row and column)
    read and written once, q, k, v read, o written, alpha and beta read:
    4096 b + 4104 bytes with fp32 scales (28,680 at b = 6), 4096 b + 3080 with
    bfloat16 ones; the two-stream kernels' own counts beside it."""
    import bench
    L, H, D, n = 2, 3, 128, 5
    p = stepq.Plan.build_uniform(0, L, H, D, bits, stepq.QUANT_DUAL_AXIS, 65536, scale_bits=scale_bits)
    rec = D * D * bits // 8 + 2 * D * (scale_bits // 8)
    assert all(p.record(l, h)[1] == rec for l in range(L) for h in range(H))
    per = 4096 * bits + (4104 if scale_bits == 32 else 3080)
    assert bench.step_bytes(p, n) == n * L * H * per
    assert bench.kernel_bytes(p, n, "fused") == n * L * H * per
    assert bench.kernel_bytes(p, n, "decode") == n * L * H * (rec + 3 * 4 * D + 8 + 2 * 4 * D)
    assert bench.kernel_bytes(p, n, "fitpack") == n * L * H * (2 * rec + 2 * 4 * D + 8)
    if bits == 6 and scale_bits == 32:
        assert per == 28680


def test_benchmark_byte_model_per_row_units():
    """Per-row (KDA) units: the gate is one alpha per key row, so a head-step
    reads 4 D + 4 gate bytes instead of 8."""
    import bench
    L, H, D, n = 1, 2, 128, 3
    p = stepq.Plan.build_uniform(1, L, H, D, 6, stepq.QUANT_DUAL_AXIS, 65536)
    rec = sum(p.record(0, h)[1] for h in range(H)) // H
    assert bench.gate_bytes(p) == 4 * D + 4
    assert bench.step_bytes(p, n) == n * L * H * (2 * rec + 3 * 4 * D + 4 * D + 4 + 4 * D)
