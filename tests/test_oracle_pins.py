"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, an invariant of the recurrence, a library routine for a special case,
brute-force enumeration, or a hand-derived byte image.  Sources: STEPQuant
paper digest page, sections 背景与动机 (update / readout / error recursion),
方法-1 (lifetime weight, allocation, pivots, bit/value), 方法-3 (dual-axis fit).
"""
import math
import os

import numpy as np
import pytest

from oracle import allocator, core, model, plan_io
from quantized_recurrent_state_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


# --------------------------------------------------------------------------
# binary16 conversion == numpy's IEEE half conversion (a library routine)
# --------------------------------------------------------------------------

def test_f16_matches_numpy():
    xs = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-9, 6, 4000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e-8, 5.96e-8, 2.98e-8, 2.99e-8,
                  6.1e-5, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11, -2.5e-7, 1e6], dtype=np.float32),
    ])
    for x in xs:
        with np.errstate(over="ignore"):
            ref = int(np.array([x], np.float32).astype(np.float16).view(np.uint16)[0])
        assert core.f32_to_f16(x) == ref, x
        back = core.f16_to_f32(ref)
        refb = float(np.array([ref], np.uint16).view(np.float16).astype(np.float32)[0])
        assert back == refb or (math.isnan(back) and math.isnan(refb))


# --------------------------------------------------------------------------
# packed format
# --------------------------------------------------------------------------

@pytest.mark.parametrize("D", [16, 128])
@pytest.mark.parametrize("b", [2, 4, 6, 8])
def test_uniform_pack_roundtrip(D, b):
    q = (1 << (b - 1)) - 1
    z = rng.integers(-q, q + 1, size=(D, D)).astype(np.int32)
    blk = core.pack_uniform(D, b, z)
    assert blk.size == D * D * b // 8
    assert np.array_equal(core.unpack_uniform(D, b, blk), z)


def test_rows_pack_roundtrip():
    D = 128
    widths = rng.choice([4, 6, 8, 16], size=D).astype(np.int32)
    z = np.zeros((D, D), np.int32)
    h = np.zeros((D, D), np.uint16)
    for i, b in enumerate(widths):
        if b == 16:
            h[i] = rng.integers(0, 1 << 16, size=D).astype(np.uint16)
        else:
            q = (1 << (b - 1)) - 1
            z[i] = rng.integers(-q, q + 1, size=D)
    blk = core.pack_rows(D, widths, z, h)
    assert blk.size == sum(D * int(b) // 8 for b in widths)
    z2, h2 = core.unpack_rows(D, widths, blk)
    assert np.array_equal(z2, z) and np.array_equal(h2, h)


def _golden_layout():
    """Cases of tests/golden/layout_uniform.txt: name -> (D, b, sets, expect)."""
    cases = {}
    with open(os.path.join(GOLDEN, "layout_uniform.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            cases.setdefault(parts[0], {})[parts[1]] = parts[2:]
    return cases


@pytest.mark.parametrize("name", ["d16b4", "d16b6", "d16b8", "d16b2", "d32b6"])
def test_uniform_layout_hand_bytes(name):
    case = _golden_layout()[name]
    D, b = int(name[1:name.index("b")]), int(name[name.index("b") + 1:])
    z = np.zeros((D, D), np.int32)
    for item in case["set"]:
        i, j, val = (int(x) for x in item.split(","))
        z[i, j] = val
    blk = core.pack_uniform(D, b, z)
    items = case["expect"]
    exp = np.full(D * D * b // 8, int(items[0].split("=")[1], 16), np.uint8)
    k = 1
    while k < len(items):
        if items[k] == "pattern":
            rng_s, pat = items[k + 1].split("=")
            a_, b_ = (int(x) for x in rng_s.split(":"))
            p = np.array([int(x, 16) for x in pat.split(",")], np.uint8)
            exp[a_:b_] = np.tile(p, (b_ - a_) // p.size)
            k += 2
        else:
            off, val = items[k].split("=")
            exp[int(off)] = int(val, 16)
            k += 1
    assert np.array_equal(blk, exp)
    assert np.array_equal(core.unpack_uniform(D, b, blk), z)


def _golden_bands():
    cases = {}
    with open(os.path.join(GOLDEN, "layout_bands.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            cases.setdefault(parts[0], {})[parts[1]] = parts[2:]
    return cases


@pytest.mark.parametrize("name", ["d16mix", "d32w8"])
def test_band_layout_hand_bytes(name):
    case = _golden_bands()[name]
    widths = np.array([int(x) for x in case["widths"][0].split(",")], np.int32)
    D = widths.size
    z = np.zeros((D, D), np.int32)
    h = np.zeros((D, D), np.uint16)
    for item in case.get("set", []):
        i, j, val = (int(x) for x in item.split(","))
        z[i, j] = val
    for item in case.get("half", []):
        i, j, val = item.split(",")
        h[int(i), int(j)] = int(val, 16)
    blk = core.pack_bands(D, widths, z, h)
    exp = np.zeros(core.codes_bytes_bands(D, widths), np.uint8)
    items = case["expect"]
    k = 0
    while k < len(items):
        if items[k] == "pattern":
            rng_s, pat = items[k + 1].split("=")
            a_, b_ = (int(x) for x in rng_s.split(":"))
            p = np.array([int(x, 16) for x in pat.split(",")], np.uint8)
            exp[a_:b_] = np.tile(p, (b_ - a_) // p.size)
            k += 2
        else:
            off, val = items[k].split("=")
            exp[int(off)] = int(val, 16)
            k += 1
    assert blk.size == exp.size
    assert np.array_equal(blk, exp)
    z2, h2 = core.unpack_bands(D, widths, blk)
    assert np.array_equal(z2, z) and np.array_equal(h2, h)


def test_band_layout_roundtrip_and_size():
    D = 128
    widths = rng.choice([2, 4, 6, 8, 16], size=D).astype(np.int32)
    z = np.zeros((D, D), np.int32)
    h = np.zeros((D, D), np.uint16)
    for i, b in enumerate(widths):
        if b == 16:
            h[i] = rng.integers(0, 1 << 16, size=D).astype(np.uint16)
        else:
            q = (1 << (b - 1)) - 1
            z[i] = rng.integers(-q, q + 1, size=D)
    blk = core.pack_bands(D, widths, z, h)
    # each band pads its tiles to whole words: between the row-major size and 31 bits per tile more
    raw = sum(D * int(b) // 8 for b in widths)
    assert raw <= blk.size < raw + 8 * 32 * 4
    assert blk.size == sum(128 * -(-int(widths[16 * g:16 * g + 16].sum()) // 8) for g in range(8))
    z2, h2 = core.unpack_bands(D, widths, blk)
    assert np.array_equal(z2, z) and np.array_equal(h2, h)


def test_rows_layout_lsb_first():
    # row-major: code j of a b-bit row occupies row bits [b*j, b*j+b)
    D = 16
    widths = np.array([4] * 8 + [2] * 8, np.int32)
    z = np.zeros((D, D), np.int32)
    z[0, 1] = 7            # u = 15 -> bits 4..7 of byte 0 (low nibble: code 0 = u 8)
    z[8, 3] = -1           # 2-bit row 8 (offset 8 rows * 8 bytes = 64), u = 1, bits 6..7
    blk = core.pack_rows(D, widths, z, np.zeros((D, D), np.uint16))
    assert blk[0] == 0xF8
    assert blk[64] == (0b10 | 0b10 << 2 | 0b10 << 4 | 0b01 << 6)


# --------------------------------------------------------------------------
# reductions
# --------------------------------------------------------------------------

def test_pairwise_sum_order_and_accuracy():
    # tree order: (1 + 0) + (2^-24 + 2^-24) = 1 + 2^-23, sequential would give 1
    assert core.pairwise_sum(np.array([1, 0, 2 ** -24, 2 ** -24], np.float32)) == np.float32(1 + 2 ** -23)
    for n in (16, 128):
        x = np.abs(rng.standard_normal(n)).astype(np.float32)
        s = float(core.pairwise_sum(x))
        exact = math.fsum(float(v) for v in x)
        assert abs(s - exact) <= math.log2(n) * 2.0 ** -24 * exact * 1.0001


def _golden_band_dot():
    cases = []
    with open(os.path.join(GOLDEN, "band_dot.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            name, D = parts[0], int(parts[1])
            x = np.full(D, float(parts[2].split("=")[1]), np.float64)
            y = np.full(D, float(parts[3].split("=")[1]), np.float64)
            cur, expect = None, None
            for tok in parts[4:]:
                if tok in ("x", "y", "expect"):
                    cur = tok
                    continue
                if cur == "expect":
                    expect = float.fromhex(tok)
                else:
                    i, val = tok.split("=")
                    (x if cur == "x" else y)[int(i)] = float.fromhex(val)
            cases.append((name, x.astype(np.float32), y.astype(np.float32), np.float32(expect)))
    return cases


@pytest.mark.parametrize("case", _golden_band_dot(), ids=lambda c: c[0])
def test_band_dot_hand_values(case):
    _, x, y, expect = case
    assert core.band_dot(x, y) == expect


@pytest.mark.parametrize("D", [16, 32, 64, 128])
def test_band_dot_exact_when_partial_sums_are(D):
    # small integers: every product and partial sum is exact, so any order gives the exact sum
    x = rng.integers(-50, 51, D).astype(np.float32)
    y = rng.integers(-50, 51, D).astype(np.float32)
    assert float(core.band_dot(x, y)) == float(np.dot(x.astype(np.int64), y.astype(np.int64)))
    # a single non-zero row picks exactly that product, wherever it sits
    for i in (0, 1, D // 2 - 1, D - 1):
        e = np.zeros(D, np.float32)
        e[i] = 3.0
        assert core.band_dot(e, y) == np.float32(3.0 * y[i])


@pytest.mark.parametrize("D", [16, 128])
def test_band_dot_error_bound(D):
    # |fl-sum - exact| <= gamma_n sum |x_i y_i|, n = RT/2 + 2 + 3 roundings on any path
    for _ in range(200):
        x = rng.standard_normal(D).astype(np.float32)
        y = (rng.standard_normal(D) * 10.0 ** rng.integers(-3, 4)).astype(np.float32)
        s = float(core.band_dot(x, y))
        exact = math.fsum(float(a) * float(b) for a, b in zip(x, y))
        n = D // 16 + 5
        bound = n * 2.0 ** -24 / (1 - n * 2.0 ** -24) * math.fsum(abs(float(a) * float(b)) for a, b in zip(x, y))
        assert abs(s - exact) <= bound


# --------------------------------------------------------------------------
# recurrence invariants (背景与动机: S_t updated by key, value, gate; readout S^T q)
# --------------------------------------------------------------------------

def _rand_inputs(D, kda=False):
    q = rng.standard_normal(D).astype(np.float32)
    n = rng.standard_normal(D)
    k = (n / np.linalg.norm(n)).astype(np.float32)
    v = rng.standard_normal(D).astype(np.float32)
    alpha = (rng.uniform(0.5, 1.0, D) if kda else np.full(D, rng.uniform(0.5, 1.0))).astype(np.float32)
    beta = np.float32(rng.uniform(0, 1))
    return q, k, v, alpha, beta


def test_fixed_point_alpha1_beta0_fp32():
    D = 128
    S = rng.standard_normal((D, D)).astype(np.float32)
    S0 = S.copy()
    q, k, v, _, _ = _rand_inputs(D)
    o = core.step_fp32(S, q, k, v, 1.0, 0.0)
    assert np.array_equal(S, S0)
    exact = (S0.astype(np.float64).T @ q.astype(np.float64))
    assert np.allclose(o, exact, rtol=1e-6, atol=1e-6)


def test_fixed_point_alpha1_beta0_from_codes():
    D = 128
    rw = np.full(D, 6, np.int32)
    S = rng.standard_normal((D, D)).astype(np.float32)
    z, h, r, c, _ = core.quantize(D, rw, np.ones(D, np.float32), np.ones(D, np.float32), S)
    q, k, v, _, _ = _rand_inputs(D)
    St, o, u, w = core.step_from_codes(D, rw, z, h, r, c, q, k, v, 1.0, 0.0)
    assert np.array_equal(St, core.reconstruct(D, rw, z, h, r, c))
    assert np.all(w == 0)


@pytest.mark.parametrize("kda", [False, True])
def test_retrieval_beta1_unit_key_fp64(kda):
    # beta = 1, ||k|| = 1: the written association is recalled exactly, S_t^T k = v,
    # for any retention (reading: Diag(alpha) acts before (I - beta k k^T)).
    D = 128
    S = rng.standard_normal((D, D))
    q, k, v, alpha, _ = _rand_inputs(D, kda)
    k64 = k.astype(np.float64)
    k64 /= np.linalg.norm(k64)
    core.step_fp64(S, q, k64, v, alpha, 1.0)
    assert np.max(np.abs(S.T @ k64 - v)) < 1e-12 * max(1.0, np.abs(v).max())


def test_pure_decay_beta0_fp64():
    D = 64
    S0 = rng.standard_normal((D, D))
    S = S0.copy()
    a = 0.97
    for t in range(50):
        q, k, v, _, _ = _rand_inputs(D)
        core.step_fp64(S, q, k, v, a, 0.0)
    assert np.allclose(S, a ** 50 * S0, rtol=1e-13, atol=0)


def test_fp32_tracks_fp64_over_256_steps():
    D = 128
    S32 = (rng.standard_normal((D, D))).astype(np.float32)
    S64 = S32.astype(np.float64)
    a = np.float32(0.995)
    worst = 0.0
    for t in range(256):
        q, k, v, _, beta = _rand_inputs(D)
        o32 = core.step_fp32(S32, q, k, v, a, beta)
        o64 = core.step_fp64(S64, q, k, v, np.float64(a), np.float64(beta))
        worst = max(worst, np.max(np.abs(o32 - o64)) / np.abs(o64).max())
    assert worst < 1e-5
    assert np.max(np.abs(S32 - S64)) < 1e-4 * max(1.0, np.abs(S64).max())


@pytest.mark.parametrize("kda", [False, True])
def test_step_from_codes_matches_fp64_update(kda):
    # the packed step equals the fp64 recurrence applied to the retained
    # reconstruction, up to the fp32 roundings of the state elements
    D = 128
    rw = np.where(rng.uniform(size=D) < 0.1, 16, 6).astype(np.int32) if kda else np.full(D, 6, np.int32)
    S = rng.standard_normal((D, D)).astype(np.float32)
    z, h, r, c, _ = core.quantize(D, rw, np.ones(D, np.float32), np.ones(D, np.float32), S)
    Shat = core.reconstruct(D, rw, z, h, r, c).astype(np.float64)
    q, k, v, alpha, beta = _rand_inputs(D, kda)
    St, o, u, w = core.step_from_codes(D, rw, z, h, r, c, q, k, v, alpha, beta)
    ref = Shat.copy()
    o_ref = core.step_fp64(ref, q, k, v, alpha.astype(np.float64), np.float64(beta))
    scale = np.abs(ref).max()
    assert np.max(np.abs(St - ref)) < 4e-6 * scale
    assert np.allclose(o, o_ref, rtol=2e-5, atol=2e-5 * scale)


@pytest.mark.parametrize("kda", [False, True])
def test_step_u_and_o_are_column_dot_products(kda):
    # u = S'^T k and o = S_t^T q column by column (not S k or S q): each within the
    # fp32 bound of the exact column dot product of the oracle's own S' and S_t
    D = 128
    rw = np.where(rng.uniform(size=D) < 0.1, 16, 6).astype(np.int32) if kda else np.full(D, 6, np.int32)
    S = (rng.standard_normal((D, D)) * rng.uniform(0.1, 10, (D, 1)) * rng.uniform(0.1, 10, (1, D))).astype(np.float32)
    z, h, r, c, _ = core.quantize(D, rw, np.ones(D, np.float32), np.ones(D, np.float32), S)
    q, k, v, alpha, beta = _rand_inputs(D, kda)
    St, o, u, w = core.step_from_codes(D, rw, z, h, r, c, q, k, v, alpha, beta)
    Shat = core.reconstruct(D, rw, z, h, r, c)
    Sp = np.where(rw[:, None] == 16, alpha[:, None] * Shat, 0).astype(np.float32)
    for i in range(D):  # S'_ij = fl(fl(alpha_i r_i) c_j) z_ij for quantized rows
        if rw[i] != 16:
            a = np.float32(alpha[i] * r[i])
            Sp[i] = (a * c).astype(np.float32) * z[i].astype(np.float32)
    k64, q64 = k.astype(np.float64), q.astype(np.float64)
    gam = 13 * 2.0 ** -24
    u_ex = Sp.astype(np.float64).T @ k64
    assert np.all(np.abs(u - u_ex) <= gam * (np.abs(Sp).astype(np.float64).T @ np.abs(k64)) + 1e-30)
    w_ex = (beta * (v - u)).astype(np.float32)
    assert np.array_equal(w, w_ex)
    assert np.array_equal(St, np.float32(Sp + k[:, None].astype(np.float64) * w[None, :].astype(np.float64)))
    o_ex = St.astype(np.float64).T @ q64
    assert np.all(np.abs(o - o_ex) <= gam * (np.abs(St).astype(np.float64).T @ np.abs(q64)) + 1e-30)
    # transposed operands would not meet the bound (the state is far from symmetric)
    assert not np.all(np.abs(o - St.astype(np.float64) @ q64) <= 1e-3 * np.abs(o_ex).max())


def test_error_recursion_and_output_error_fp64():
    # E_t = A_t E_{t-1} + eps_t and output error = E_{t-1}^T A_t^T q_t
    # (背景与动机).  Quantized trajectory: exact update of the reconstructed
    # state, then requantization (eps_t = S_hat_t - S_tilde_t).
    D = 128
    rw = np.full(D, 4, np.int32)
    ones = np.ones(D, np.float32)
    S_fp = rng.standard_normal((D, D))
    S_hat = S_fp.copy()
    E = S_hat - S_fp
    for t in range(24):
        q, k, v, alpha, beta = _rand_inputs(D, kda=True)
        a64, b64 = alpha.astype(np.float64), np.float64(beta)
        o_fp = core.step_fp64(S_fp, q, k, v, a64, b64)
        S_tilde = S_hat.copy()
        o_q = core.step_fp64(S_tilde, q, k, v, a64, b64)
        AE = E.copy()
        o_err = core.step_fp64(AE, q, k, np.zeros(D), a64, b64)   # A_t E_{t-1}, (A_t E)^T q
        z, h, r, c, _ = core.quantize(D, rw, ones, ones, S_tilde.astype(np.float32))
        S_new = r.astype(np.float64)[:, None] * c.astype(np.float64)[None, :] * z
        eps = S_new - S_tilde
        S_hat = S_new
        E_new = S_hat - S_fp
        scale = np.abs(E_new).max()
        assert np.max(np.abs(E_new - (AE + eps))) <= 1e-12 * max(scale, np.abs(S_fp).max())
        assert np.max(np.abs((o_q - o_fp) - o_err)) <= 1e-11 * np.abs(o_fp).max()
        E = E_new


# --------------------------------------------------------------------------
# lifetime weight (方法-1)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("h", [2.0, 50.0, 1000.0, 20000.0])
def test_lifetime_closed_form(h):
    l = -math.log(2.0) / h
    H = 4096
    assert math.isclose(core.lifetime_weight(l, H), allocator.lifetime_weight_closed_form(l, H), rel_tol=1e-12)
    assert core.lifetime_weight(0.0, 100) == 100.0


# --------------------------------------------------------------------------
# quantizer (方法-3)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("b", [2, 4, 6, 8])
def test_quantizer_constant_magnitude(b):
    D = 128
    s = np.float32(0.25)
    S = (s * np.where(rng.uniform(size=(D, D)) < 0.5, -1, 1)).astype(np.float32)
    rw = np.full(D, b, np.int32)
    ones = np.ones(D, np.float32)
    z, h, r, c, tie = core.quantize(D, rw, ones, ones, S)
    q = (1 << (b - 1)) - 1
    assert np.array_equal(np.abs(z), np.full((D, D), q))
    assert np.array_equal(np.sign(z), np.sign(S).astype(np.int32))
    Sh = core.reconstruct(D, rw, z, h, r, c)
    assert np.max(np.abs(Sh - S)) <= 2 * np.spacing(s)


@pytest.mark.parametrize("b", [2, 4, 6, 8])
def test_quantizer_half_step_bound(b):
    D = 128
    S = (rng.standard_normal((D, D)) * rng.uniform(0.1, 10, (D, 1)) * rng.uniform(0.1, 19, (1, D))).astype(np.float32)
    rw = np.full(D, b, np.int32)
    wbar = rng.uniform(0.2, 5.0, D).astype(np.float32)
    rho = (1.0 / np.sqrt(np.sqrt(wbar.astype(np.float64)))).astype(np.float32)
    z, h, r, c, tie = core.quantize(D, rw, rho, wbar, S)
    q = (1 << (b - 1)) - 1
    assert np.abs(z).max() <= q
    Sh = core.reconstruct(D, rw, z, h, r, c).astype(np.float64)
    step = r.astype(np.float64)[:, None] * c.astype(np.float64)[None, :]
    unclamped = np.abs(z) < q
    err = np.abs(Sh - S)
    bound = 0.5 * step * (1 + 1e-5) + 2 * np.spacing(np.abs(S.astype(np.float32)))
    assert np.all(err[unclamped] <= bound[unclamped])


def test_quantizer_refinement_is_weighted_ls():
    # for the initial codes z0, c_j minimises sum_i w_i (S_ij - r_i c z0_ij)^2
    D = 128
    b = 4
    S = (rng.standard_normal((D, D)) * rng.uniform(0.5, 3, (D, 1))).astype(np.float32)
    rw = np.full(D, b, np.int32)
    wbar = rng.uniform(0.2, 5.0, D).astype(np.float32)
    rho = (1.0 / np.sqrt(np.sqrt(wbar.astype(np.float64)))).astype(np.float32)
    z, h, r, c, tie, z0 = core.quantize(D, rw, rho, wbar, S, return_z0=True)
    S64, r64, w64 = S.astype(np.float64), r.astype(np.float64), wbar.astype(np.float64)
    invphi = (math.sqrt(5) - 1) / 2
    for j in range(0, D, 7):
        f = lambda cc: float(np.sum(w64 * (S64[:, j] - r64 * cc * z0[:, j]) ** 2))
        lo, hi = 0.2 * c[j], 5.0 * c[j]
        x1, x2 = hi - invphi * (hi - lo), lo + invphi * (hi - lo)
        f1, f2 = f(x1), f(x2)
        for _ in range(120):
            if f1 < f2:
                hi, x2, f2 = x2, x1, f1
                x1 = hi - invphi * (hi - lo)
                f1 = f(x1)
            else:
                lo, x1, f1 = x1, x2, f2
                x2 = lo + invphi * (hi - lo)
                f2 = f(x2)
        assert math.isclose(c[j], 0.5 * (lo + hi), rel_tol=1e-5)


def test_quantizer_scale_invariance():
    # S -> 2^k S scales the row factors by 2^k and leaves c and z unchanged
    D = 128
    S = rng.standard_normal((D, D)).astype(np.float32)
    rw = np.full(D, 6, np.int32)
    wbar = rng.uniform(0.2, 5.0, D).astype(np.float32)
    rho = (1.0 / np.sqrt(np.sqrt(wbar.astype(np.float64)))).astype(np.float32)
    z1, _, r1, c1, _ = core.quantize(D, rw, rho, wbar, S)
    z2, _, r2, c2, _ = core.quantize(D, rw, rho, wbar, (S * np.float32(8.0)).astype(np.float32))
    assert np.array_equal(z1, z2) and np.array_equal(c1, c2) and np.array_equal(r2, r1 * 8)


def test_quantizer_degenerate():
    D = 16
    rw = np.full(D, 4, np.int32)
    ones = np.ones(D, np.float32)
    S = np.zeros((D, D), np.float32)
    z, h, r, c, _ = core.quantize(D, rw, ones, ones, S)
    assert np.all(z == 0) and np.all(c == 1.0) and np.all(r == np.float32(1e-12))
    S = rng.standard_normal((D, D)).astype(np.float32)
    S[:, 3] = 0
    z, h, r, c, _ = core.quantize(D, rw, ones, ones, S)
    assert c[3] == 1.0 and np.all(z[:, 3] == 0)


def test_quantizer_pivot_rows_fp16():
    D = 16
    rw = np.array([4] * 12 + [16] * 4, np.int32)
    ones = np.ones(D, np.float32)
    S = rng.standard_normal((D, D)).astype(np.float32)
    z, h, r, c, _ = core.quantize(D, rw, ones, ones, S)
    assert np.array_equal(h[12:], S[12:].astype(np.float16).view(np.uint16))
    assert np.all(r[12:] == 0)
    # the pivot rows take no part in the column fit: same c as without them
    z2, _, _, c2, _ = core.quantize(D, rw[:12].tolist() + [16] * 4, ones, ones,
                                    np.concatenate([S[:12], np.zeros((4, D), np.float32)]))
    assert np.array_equal(c, c2)


def test_tie_flag():
    # a value placed on a .5 boundary is flagged
    D = 16
    rw = np.full(D, 2, np.int32)
    ones = np.ones(D, np.float32)
    S = np.ones((D, D), np.float32)
    S[0, 0] = 0.5       # with r = mean|S| ~ 1, c = 1: x = 0.5 / r ... near .5 boundary
    z, h, r, c, tie = core.quantize(D, rw, ones, ones, S)
    y = (S * (np.float32(1) / r)[:, None]).astype(np.float32)
    x = y.astype(np.float64) * (np.float32(1) / c).astype(np.float64)[None, :]
    frac = np.abs(np.abs(x) - (np.floor(np.abs(x)) + 0.5))
    assert np.array_equal(tie & 1, (frac <= 1e-6 * np.abs(x)).astype(np.uint8))


# --------------------------------------------------------------------------
# allocator (方法-1)
# --------------------------------------------------------------------------

def _convex_costs(N, widths):
    # d(b) decreasing and convex in b, times a lifetime weight
    out = np.zeros((N, len(widths)))
    for u in range(N):
        base = rng.uniform(0.5, 2.0)
        rate = rng.uniform(0.3, 0.7)
        Lw = rng.uniform(1.0, 100.0)
        out[u] = Lw * base * np.exp(-rate * np.asarray(widths, float))
    return out


# --------------------------------------------------------------------------
# per-row absmax baseline quantizer (实验: uniform INT-b, ordinary per-row
# absmax): nearest code by enumeration, the row maximum at +-qmax, the
# half-step bound, c = 1, degenerate rows, scale invariance
# --------------------------------------------------------------------------

def _outlier_state(D, seed):
    g = np.random.default_rng(seed)
    S = g.standard_normal((D, D)).astype(np.float32)
    S[g.integers(D)] *= 10.0
    S[:, g.integers(D)] *= 19.0
    return S


# --------------------------------------------------------------------------
# 16-bit (bfloat16) scale storage: the conversion against torch's bfloat16,
# r = bf16(r of the fp32 fit), codes nearest to y * fl(1/c) with the stored
# scales, the half-step bound with the stored scales, record bytes
# --------------------------------------------------------------------------

def test_bf16_matches_torch():
    torch = pytest.importorskip("torch")
    xs = np.concatenate([
        rng.standard_normal(5000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 5000),
        np.array([0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, 3e38, 1e-40, -2.5], np.float32),
    ]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for x, rb in zip(xs, ref):
        assert core.f32_to_bf16(x) == int(rb), x
        assert core.bf16_to_f32(int(rb)) == float(torch.tensor([int(rb)], dtype=torch.int32).to(torch.int16)
                                                   .view(torch.bfloat16).float()[0])


@pytest.mark.parametrize("b", [4, 6, 8])
def test_scale16_rows_are_rounded_fp32_rows_and_codes_nearest(b):
    torch = pytest.importorskip("torch")
    D, q = 16, (1 << (b - 1)) - 1
    S = _outlier_state(D, 500 + b)
    widths = np.full(D, b)
    rho = np.linspace(0.7, 1.3, D).astype(np.float32)
    wbar = (1.0 / rho.astype(np.float64) ** 4).astype(np.float32)
    z32, _, r32, c32, _ = core.quantize(D, widths, rho, wbar, S)
    z16, _, r16, c16, _ = core.quantize(D, widths, rho, wbar, S, scale_bits=16)
    bf = torch.from_numpy(r32).to(torch.bfloat16).float().numpy()
    assert np.array_equal(r16, bf)
    for x in np.concatenate([r16, c16]):  # representable in bfloat16
        assert np.float32(x).view(np.uint32) & 0xFFFF == 0
    cand = np.arange(-q, q + 1, dtype=np.float64)
    for i in range(D):
        inv_r = np.float32(1.0) / r16[i]
        for j in range(D):
            y = np.float32(S[i, j] * inv_r)
            x = float(y) * float(np.float32(1.0) / c16[j])
            dd = np.abs(cand - x)
            best = cand[dd == dd.min()]
            pick = best[0] if best.size == 1 else best[np.argmin(np.abs(best) % 2)]
            assert z16[i, j] == int(pick), (i, j)
            if abs(x) <= q:
                assert abs(float(S[i, j]) - float(r16[i]) * float(c16[j]) * z16[i, j]) <= \
                    0.5 * float(r16[i]) * float(c16[j]) * (1 + 1e-5) + 1e-6 * abs(float(S[i, j]))


def test_scale16_record_layout_and_plan_field(tmp_path):
    D = 16
    plan = model.uniform_plan(0, D, 2, 2, 6, model.QUANT_DUAL_AXIS, 4096, scale_bits=16)
    back = plan_io.read_plan(plan_io.write_plan(str(tmp_path / "p.bin"), plan))
    assert back["scale_bits"] == 16
    assert plan_io.record_bytes(0, D, np.full(D, 6), 16) == 256  # 192 code bytes + 64 scale bytes
    assert plan_io.record_bytes(0, 128, np.full(128, 6), 16) == 12288 + 512
    pv = model.PlanView(back)
    slot = np.zeros(pv.slot_bytes, np.uint8)
    S = _outlier_state(D, 600)
    pv.quantize_into(slot, 1, 1, S)
    z, h, r, c = pv.unpack(slot, 1, 1)
    z2, _, r2, c2, _ = core.quantize(D, np.full(D, 6), pv.rho[1, 1], pv.wbar[1, 1], S, scale_bits=16)
    assert np.array_equal(z, z2) and np.array_equal(r, r2) and np.array_equal(c, c2)


@pytest.mark.parametrize("b", [2, 4, 6, 8])
def test_absmax_codes_are_nearest_by_enumeration(b):
    D, q = 16, (1 << (b - 1)) - 1
    S = _outlier_state(D, 100 + b)
    z, h, r, c, tie = core.quantize_absmax(D, np.full(D, b), S)
    assert np.all(c == 1.0)
    cand = np.arange(-q, q + 1, dtype=np.float64)
    for i in range(D):
        m = float(np.max(np.abs(S[i])))
        assert abs(float(r[i]) * q - m) <= 2.0 ** -23 * m  # r_i is m_i / qmax rounded once
        inv = np.float32(1.0) / r[i]
        for j in range(D):
            x = float(S[i, j]) * float(inv)
            d = np.abs(cand - x)
            best = cand[d == d.min()]
            pick = best[0] if best.size == 1 else best[np.argmin(np.abs(best) % 2)]  # ties to even
            assert z[i, j] == int(pick), (i, j, x)


@pytest.mark.parametrize("b", [2, 4, 6, 8])
def test_absmax_row_max_at_qmax_and_half_step(b):
    D, q = 128, (1 << (b - 1)) - 1
    S = _outlier_state(D, 200 + b)
    z, h, r, c, tie = core.quantize_absmax(D, np.full(D, b), S)
    jmax = np.argmax(np.abs(S), axis=1)
    assert np.all(np.abs(z[np.arange(D), jmax]) == q)
    assert np.all(np.sign(z[np.arange(D), jmax]) == np.sign(S[np.arange(D), jmax]))
    err = np.abs(S.astype(np.float64) - r[:, None].astype(np.float64) * z)
    assert np.all(err <= 0.5 * r[:, None] * (1 + 1e-5))


def test_absmax_degenerate_and_scale_invariance():
    D, b = 16, 6
    S = _outlier_state(D, 300)
    S[3] = 0.0
    z, h, r, c, tie = core.quantize_absmax(D, np.full(D, b), S)
    assert r[3] == 1.0 and np.all(z[3] == 0)
    z2, h2, r2, c2, tie2 = core.quantize_absmax(D, np.full(D, b), S * np.float32(2.0 ** 7))
    assert np.array_equal(z2, z)
    nz = np.arange(D) != 3
    assert np.array_equal(r2[nz], r[nz] * np.float32(2.0 ** 7))


def test_absmax_pivot_rows_fp16_and_plan_field(tmp_path):
    D = 16
    S = _outlier_state(D, 400)
    widths = np.full(D, 6)
    widths[[2, 9]] = model.PIVOT_BITS
    z, h, r, c, tie = core.quantize_absmax(D, widths, S)
    for i in (2, 9):
        assert r[i] == 0.0 and np.all(z[i] == 0)
        assert np.array_equal(h[i], S[i].astype(np.float16).view(np.uint16))
    plan = model.uniform_plan(0, D, 2, 3, 4, model.QUANT_ABSMAX, 65536)
    back = plan_io.read_plan(plan_io.write_plan(str(tmp_path / "p.bin"), plan))
    assert back["quantizer"] == model.QUANT_ABSMAX and np.all(back["widths"] == 4)
    # a decode step through the plan view keeps c = 1 in the record
    pv = model.PlanView(back)
    slot = np.zeros(pv.slot_bytes, np.uint8)
    pv.quantize_into(slot, 1, 2, S)
    g = np.random.default_rng(5)
    k = g.standard_normal(D).astype(np.float32)
    k /= np.linalg.norm(k)
    pv.step(slot, 1, 2, g.standard_normal(D).astype(np.float32), k, g.standard_normal(D).astype(np.float32),
            np.full(D, 0.9, np.float32), np.float32(0.5))
    zz, hh, rr, cc = pv.unpack(slot, 1, 2)
    assert np.all(cc == 1.0) and np.all(np.abs(zz) <= 7)


@pytest.mark.parametrize("widths", [(4, 6, 8), (2, 4, 6, 8)])
@pytest.mark.parametrize("N", [3, 5, 7])
def test_dp_equals_brute_force(widths, N):
    for trial in range(6):
        cost = rng.uniform(0, 10, (N, len(widths)))   # arbitrary (non-convex too)
        for nominal in (widths[0] + 0.5, (widths[0] + widths[-1]) / 2, widths[-1] - 1.0):
            cap = allocator.budget_cap(nominal, N)
            a = allocator.dp_allocate_budget(cost, widths, cap)
            bf = allocator.brute_force(cost, widths, cap)
            assert np.array_equal(a, bf)
            assert a.sum() <= cap


@pytest.mark.parametrize("widths", [(4, 6, 8), (2, 4, 6, 8)])
@pytest.mark.parametrize("N", [4, 6, 8])
def test_lagrangian_equals_brute_force_convex(widths, N):
    for trial in range(6):
        cost = _convex_costs(N, widths)
        for nominal in (widths[0] + 0.7, (widths[0] + widths[-1]) / 2, widths[-1] - 0.6):
            cap = allocator.budget_cap(nominal, N)
            a = allocator.lagrangian_allocate(cost, widths, cap)
            bf = allocator.brute_force(cost, widths, cap)
            assert a.sum() <= cap
            assert math.isclose(allocator.total_cost(cost, widths, a),
                                allocator.total_cost(cost, widths, bf), rel_tol=1e-12)


def test_lagrangian_nonconvex_gap_reported():
    widths = (4, 6, 8)
    gaps = []
    for trial in range(20):
        cost = rng.uniform(0, 10, (6, 3))
        cap = allocator.budget_cap(6.0, 6)
        a = allocator.lagrangian_allocate(cost, widths, cap)
        bf = allocator.brute_force(cost, widths, cap)
        assert a.sum() <= cap
        ca, cb = allocator.total_cost(cost, widths, a), allocator.total_cost(cost, widths, bf)
        assert ca >= cb - 1e-12
        gaps.append(ca / cb - 1)
    print("non-convex Lagrangian gap: max %.3g mean %.3g" % (max(gaps), float(np.mean(gaps))))


def test_pivots_top_scores_ties_lower_index():
    L = np.array([1.0, 2.0, 2.0, 0.5, 3.0])
    d = np.array([1.0, 1.0, 1.0, 1.0, 1.0])
    assert list(allocator.select_pivots(L, d, 2)) == [1, 4]
    assert list(allocator.select_pivots(L, d, 3)) == [1, 2, 4]


def test_bits_per_value_hand_count():
    # mode 0, D = 16, two heads at widths 4 and 16 (pivot):
    # codes 4*256 + 16*256 = 5120; scales of head 0: (16 + 16) * 32 = 1024 -> 6144 / 512
    assert allocator.bits_per_value(0, 1, 2, 16, [4, 16]) == 12.0
    # mode 1, D = 16, one head: 15 rows at 4 bits and 1 FP16 row:
    # codes 15*16*4 + 16*16 = 1216; r 15*32 = 480; c 16*32 = 512 -> 2208 / 256
    assert allocator.bits_per_value(1, 1, 1, 16, [4] * 15 + [16]) == 2208 / 256
    # 16-bit scale accounting of the same head
    assert allocator.bits_per_value(1, 1, 1, 16, [4] * 15 + [16], scale_bits=16) == (1216 + 15 * 16 + 256) / 256


def test_real_distortion_curves_are_convex():
    # the quantizer's distortion falls convexly with the width on this data,
    # which is what makes the Lagrangian + repair exact
    D = 128
    S = (rng.standard_normal((D, D)) * rng.uniform(0.5, 3, (D, 1))).astype(np.float32)
    ones = np.ones(D, np.float32)
    d = [core.distortion_rows(D, b, ones, ones, S).sum() for b in (2, 4, 6, 8)]
    drops = -np.diff(d)
    assert np.all(drops > 0) and np.all(np.diff(drops) < 0)


def test_plan_roundtrip(tmp_path):
    wl = synth.workloads()["tiny_gdn"]
    D = wl.d
    plan = dict(mode=0, n_layers=1, n_heads=4, d=D, n_pivots=1, bitset=[2, 4, 6], nominal_bits=4.0,
                horizon=65536, widths=np.array([2, 6, 16, 4], np.uint8),
                wbar=np.ones(4 * D, np.float32), rho=np.ones(4 * D, np.float32),
                lgate=np.zeros(4), lifetime=np.ones(4))
    data = plan_io.write_plan(str(tmp_path / "p.bin"), plan)
    back = plan_io.read_plan(data)
    assert np.array_equal(back["widths"], plan["widths"]) and back["mode"] == 0
    offs, slot = plan_io.pool_layout(back)
    # records: b=2: 64+128 -> 256; b=6: 192+128 -> 384; pivot 512; b=4: 128+128 = 256
    assert list(offs) == [0, 256, 640, 1152] and slot == 1408


# --------------------------------------------------------------------------
# chunked prefill: the chunk formulas equal the sequential recurrence (fp64),
# for ragged lengths and any chunk size; a one-token chunk is one step
# --------------------------------------------------------------------------

def _prompt(T, D, seed):
    g = np.random.default_rng(seed)
    Q = g.standard_normal((T, D))
    K = g.standard_normal((T, D))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = g.standard_normal((T, D))
    alpha = np.exp(-np.log(2) / np.exp(g.uniform(np.log(2), np.log(2000), T)))
    beta = g.uniform(0, 1, T)
    S0 = g.standard_normal((D, D))
    return S0, Q, K, V, alpha, beta


@pytest.mark.parametrize("T,C", [(1, 64), (63, 64), (64, 64), (65, 64), (200, 64), (130, 16), (37, 8)])
def test_chunked_prefill_equals_sequential(T, C):
    from oracle import prefill
    S0, Q, K, V, alpha, beta = _prompt(T, 32, 700 + T + C)
    O_seq, S_seq = prefill.sequential(S0, Q, K, V, alpha, beta)
    O_chk, S_chk = prefill.chunked(S0, Q, K, V, alpha, beta, C)
    assert np.max(np.abs(O_chk - O_seq)) <= 1e-11 * max(1.0, np.max(np.abs(O_seq)))
    assert np.max(np.abs(S_chk - S_seq)) <= 1e-11 * max(1.0, np.max(np.abs(S_seq)))


def test_chunk_of_one_token_is_one_step():
    from oracle import prefill
    S0, Q, K, V, alpha, beta = _prompt(1, 16, 9)
    O, S = prefill.chunk(S0, Q, K, V, alpha, beta)
    S_ref = alpha[0] * S0 + beta[0] * np.outer(K[0], V[0] - alpha[0] * S0.T @ K[0])
    assert np.allclose(S, S_ref, rtol=1e-14, atol=1e-14)
    assert np.allclose(O[0], S_ref.T @ Q[0], rtol=1e-13, atol=1e-13)


def _prompt_rows(T, D, seed):
    S0, Q, K, V, _, beta = _prompt(T, D, seed)
    g = np.random.default_rng(seed + 1)
    alpha = np.exp(-np.log(2) / np.exp(g.uniform(np.log(2), np.log(2000), (T, D))))
    return S0, Q, K, V, alpha, beta


@pytest.mark.parametrize("T,C", [(1, 64), (64, 64), (65, 64), (150, 64), (37, 8)])
def test_chunked_prefill_rows_equals_sequential(T, C):
    # per-key-row gates: the chunk form against the token-by-token recurrence
    from oracle import prefill
    S0, Q, K, V, alpha, beta = _prompt_rows(T, 32, 900 + T + C)
    O_seq, S_seq = prefill.sequential(S0, Q, K, V, alpha, beta)
    O_chk, S_chk = prefill.chunked_rows(S0, Q, K, V, alpha, beta, C)
    assert np.max(np.abs(O_chk - O_seq)) <= 1e-11 * max(1.0, np.max(np.abs(O_seq)))
    assert np.max(np.abs(S_chk - S_seq)) <= 1e-11 * max(1.0, np.max(np.abs(S_seq)))


def test_chunked_prefill_rows_with_equal_gates_is_the_scalar_form():
    # a gate that is the same for every key row reduces to the per-head chunk form
    from oracle import prefill
    S0, Q, K, V, alpha, beta = _prompt(70, 16, 31)
    rows = np.repeat(alpha[:, None], 16, axis=1)
    O1, S1 = prefill.chunked(S0, Q, K, V, alpha, beta)
    O2, S2 = prefill.chunked_rows(S0, Q, K, V, rows, beta)
    assert np.allclose(O1, O2, rtol=1e-12, atol=1e-12) and np.allclose(S1, S2, rtol=1e-12, atol=1e-12)


def test_chunk_rows_of_one_token_is_the_gated_step():
    # one token: S_1 = (I - beta k k^T) Diag(alpha) S_0 + beta k v^T written out
    from oracle import prefill
    S0, Q, K, V, alpha, beta = _prompt_rows(1, 12, 5)
    O, S = prefill.chunk_rows(S0, Q, K, V, alpha, beta)
    k = K[0]
    S_ref = (np.eye(12) - beta[0] * np.outer(k, k)) @ (alpha[0][:, None] * S0) + beta[0] * np.outer(k, V[0])
    assert np.allclose(S, S_ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(O[0], S_ref.T @ Q[0], rtol=1e-13, atol=1e-13)
