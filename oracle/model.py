"""Head-, pool- and plan-level oracle built on the C oracle -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg use it.

Source: STEPQuant paper digest page (vibe-research): 方法-1 (calibration
statistics, lifetime weight, allocation, FP16 pivots), 方法-2 (row impact
g_t = A_t^T q_t, omega_i = E[g_{t,i}^2]), 方法-3 (dual-axis fit), 方法-4
(per-step order: reconstruct, update + readout, refit, pack).
"""
from __future__ import annotations

import math

import numpy as np

from . import allocator, core, plan_io

PIVOT_BITS = 16


# --------------------------------------------------------------------------
# one head
# --------------------------------------------------------------------------

def _scales_to_bytes(x, scale_bits):
    x = np.asarray(x, dtype=np.float32)
    if scale_bits == 16:
        return np.array([core.f32_to_bf16(float(v)) for v in x], dtype="<u2").view(np.uint8)
    return x.astype("<f4").view(np.uint8)


def _scales_from_bytes(b, D, scale_bits):
    if scale_bits == 16:
        return np.array([core.bf16_to_f32(int(v)) for v in b[:2 * D].view("<u2")], dtype=np.float32)
    return b[:4 * D].view("<f4").astype(np.float32)


def pack_head(mode: int, D: int, rw, z, h, r, c, scale_bits: int = 32) -> np.ndarray:
    rw = np.asarray(rw, dtype=np.int32)
    rec = np.zeros(plan_io.record_bytes(mode, D, rw, scale_bits), dtype=np.uint8)
    if mode == 0 and rw[0] == PIVOT_BITS:
        blk = core.pack_rows(D, rw, np.zeros((D, D), np.int32), h)
        rec[:blk.size] = blk
        return rec
    if mode == 0:
        blk = core.pack_uniform(D, int(rw[0]), z)
    else:
        blk = core.pack_bands(D, rw, z, h)
    rec[:blk.size] = blk
    e = scale_bits // 8
    rec[blk.size:blk.size + e * D] = _scales_to_bytes(r, scale_bits)
    rec[blk.size + e * D:blk.size + 2 * e * D] = _scales_to_bytes(c, scale_bits)
    return rec


def unpack_head(mode: int, D: int, rw, rec: np.ndarray, scale_bits: int = 32):
    rw = np.asarray(rw, dtype=np.int32)
    rec = np.ascontiguousarray(rec, dtype=np.uint8)
    nb = plan_io.codes_block_bytes(mode, D, rw)
    if mode == 0 and rw[0] == PIVOT_BITS:
        z, h = core.unpack_rows(D, rw, rec[:nb])
        return z, h, np.zeros(D, np.float32), np.zeros(D, np.float32)
    if mode == 0:
        z = core.unpack_uniform(D, int(rw[0]), rec[:nb])
        h = np.zeros((D, D), np.uint16)
    else:
        z, h = core.unpack_bands(D, rw, rec[:nb])
    e = scale_bits // 8
    r = _scales_from_bytes(rec[nb:nb + e * D], D, scale_bits)
    c = _scales_from_bytes(rec[nb + e * D:nb + 2 * e * D], D, scale_bits)
    return z, h, r, c


QUANT_DUAL_AXIS = 0  # STEPQuant row/column fit (方法-3)
QUANT_ABSMAX = 1     # ordinary per-row absmax baseline (实验)


def quantize_head(mode, D, rw, rho, wbar, S, quantizer: int = QUANT_DUAL_AXIS, scale_bits: int = 32):
    if quantizer == QUANT_ABSMAX:
        z, h, r, c, tie = core.quantize_absmax(D, rw, S, scale_bits=scale_bits)
    else:
        z, h, r, c, tie = core.quantize(D, rw, rho, wbar, S, scale_bits=scale_bits)
    return pack_head(mode, D, rw, z, h, r, c, scale_bits), tie


def reconstruct_head(mode, D, rw, rec, scale_bits: int = 32):
    z, h, r, c = unpack_head(mode, D, rw, rec, scale_bits)
    return core.reconstruct(D, rw, z, h, r, c)


def step_head(mode, D, rw, rho, wbar, rec, q, k, v, alpha, beta, quantizer: int = QUANT_DUAL_AXIS,
              scale_bits: int = 32):
    """Decode step of one packed head.  Returns (new record, o, tie, S_t, w)."""
    z, h, r, c = unpack_head(mode, D, rw, rec, scale_bits)
    S, o, u, w = core.step_from_codes(D, rw, z, h, r, c, q, k, v, alpha, beta)
    new_rec, tie = quantize_head(mode, D, rw, rho, wbar, S, quantizer, scale_bits)
    return new_rec, o, tie, S, w


# --------------------------------------------------------------------------
# plan-level helpers
# --------------------------------------------------------------------------

class PlanView:
    """Per-head metadata of a plan dict (as returned by plan_io.read_plan)."""

    def __init__(self, plan: dict):
        self.plan = plan
        self.mode = int(plan["mode"])
        self.L = int(plan["n_layers"])
        self.H = int(plan["n_heads"])
        self.D = int(plan["d"])
        self.offsets, self.slot_bytes = plan_io.pool_layout(plan)
        self.rho = np.asarray(plan["rho"], np.float32).reshape(self.L, self.H, self.D)
        self.wbar = np.asarray(plan["wbar"], np.float32).reshape(self.L, self.H, self.D)
        self.quantizer = int(plan.get("quantizer", QUANT_DUAL_AXIS))
        self.scale_bits = int(plan.get("scale_bits", 32))

    def rw(self, l, h):
        return plan_io.head_row_widths(self.plan, l, h)

    def rec_bytes(self, l, h):
        return plan_io.record_bytes(self.mode, self.D, self.rw(l, h), self.scale_bits)

    def record(self, pool_slot: np.ndarray, l, h):
        o = int(self.offsets[l * self.H + h])
        return pool_slot[o:o + self.rec_bytes(l, h)]

    def quantize_into(self, pool_slot: np.ndarray, l, h, S):
        rec, tie = quantize_head(self.mode, self.D, self.rw(l, h), self.rho[l, h], self.wbar[l, h], S,
                                 self.quantizer, self.scale_bits)
        o = int(self.offsets[l * self.H + h])
        pool_slot[o:o + rec.size] = rec
        return tie

    def step(self, pool_slot: np.ndarray, l, h, q, k, v, alpha, beta):
        """Step one (slot, layer, head) in place; returns (o, tie, S_t, w)."""
        rec = self.record(pool_slot, l, h).copy()
        new_rec, o, tie, S, w = step_head(self.mode, self.D, self.rw(l, h), self.rho[l, h],
                                          self.wbar[l, h], rec, q, k, v, alpha, beta, self.quantizer,
                                          self.scale_bits)
        off = int(self.offsets[l * self.H + h])
        pool_slot[off:off + new_rec.size] = new_rec
        return o, tie, S, w

    def unpack(self, pool_slot, l, h):
        return unpack_head(self.mode, self.D, self.rw(l, h), self.record(pool_slot, l, h), self.scale_bits)

    def reconstruct(self, pool_slot, l, h):
        return reconstruct_head(self.mode, self.D, self.rw(l, h), self.record(pool_slot, l, h), self.scale_bits)


# --------------------------------------------------------------------------
# calibration and planning (方法-1, 方法-2)
# --------------------------------------------------------------------------

def calibrate(mode: int, D: int, n_layers: int, n_heads: int, S0, steps, bits,
              snapshot_every: int = 8):
    """Run the FP32 recurrence on calibration inputs and collect the statistics.

    S0: [n_req, L, H, D, D] float32.  steps: iterable of dicts with q, k, v
    ([n_req, L, H, D]), alpha ([n_req, L, H] or [n_req, L, H, D]) and beta
    ([n_req, L, H]).  Returns wbar, rho ([L, H, D]), lgate and the distortion
    table d[u, m] for the units of `mode`.

    omega_i = mean over steps and requests of g_i^2 with g = A_t^T q_t; the
    plan stores wbar_i = omega_i / mean_i omega_i (floored at 1e-12) and
    rho_i = wbar_i^(-1/4) = 1/sqrt(sqrt(wbar_i)).  l_u = mean log gate.
    d_u(b) = mean over snapshots (every `snapshot_every`-th step) of the
    squared Frobenius error of the unit when its head is quantized at b."""
    steps = list(steps)
    S = np.array(S0, dtype=np.float32, copy=True)
    n_req = S.shape[0]
    omega = np.zeros((n_layers, n_heads, D))
    lsum = np.zeros((n_layers, n_heads, D))
    count = 0
    for st in steps:
        for n in range(n_req):
            for l in range(n_layers):
                for h in range(n_heads):
                    al = _alpha_rows(st["alpha"][n, l, h], D)
                    om = omega[l, h]
                    ls = lsum[l, h]
                    core.calib_accumulate(st["q"][n, l, h], st["k"][n, l, h], al, st["beta"][n, l, h], om, ls)
        count += 1
    omega /= (count * n_req)
    lmean = lsum / (count * n_req)
    mean_om = omega.mean(axis=2, keepdims=True)
    wbar64 = np.maximum(omega / mean_om, 1e-12)
    wbar = wbar64.astype(np.float32)
    rho = (1.0 / np.sqrt(np.sqrt(wbar.astype(np.float64)))).astype(np.float32)

    dist_rows = np.zeros((n_layers, n_heads, D, len(bits)))
    n_snap = 0
    for t, st in enumerate(steps):
        for n in range(n_req):
            for l in range(n_layers):
                for h in range(n_heads):
                    al = _alpha_rows(st["alpha"][n, l, h], D)
                    core.step_fp32(S[n, l, h], st["q"][n, l, h], st["k"][n, l, h], st["v"][n, l, h],
                                   al, st["beta"][n, l, h])
        if (t + 1) % snapshot_every == 0:
            n_snap += 1
            for n in range(n_req):
                for l in range(n_layers):
                    for h in range(n_heads):
                        for m, b in enumerate(bits):
                            dist_rows[l, h, :, m] += core.distortion_rows(D, b, rho[l, h], wbar[l, h], S[n, l, h])
    dist_rows /= max(1, n_snap * n_req)
    if mode == 0:
        dist = dist_rows.sum(axis=2).reshape(n_layers * n_heads, len(bits))
        lgate = lmean.mean(axis=2).reshape(-1)
    else:
        dist = dist_rows.reshape(n_layers * n_heads * D, len(bits))
        lgate = lmean.reshape(-1)
    return dict(wbar=wbar, rho=rho, lgate=lgate, dist=dist)


def _alpha_rows(a, D):
    a = np.asarray(a, dtype=np.float32)
    return np.full(D, a, np.float32) if a.ndim == 0 else a


def build_plan(mode: int, D: int, n_layers: int, n_heads: int, stats: dict, bits,
               nominal_bits: float, n_pivots: int, horizon: int, lifetime=None, scale_bits: int = 32) -> dict:
    """Pivots, then DP (mode 0) or Lagrangian + repair (mode 1) allocation."""
    lgate = np.asarray(stats["lgate"], dtype=np.float64)
    if lifetime is None:
        lifetime = np.array([core.lifetime_weight(float(l), horizon) for l in lgate])
    dist = np.asarray(stats["dist"], dtype=np.float64)
    bits = sorted(int(b) for b in bits)
    n_units = lgate.size
    piv = allocator.select_pivots(lifetime, dist[:, -1], n_pivots)
    keep = np.setdiff1d(np.arange(n_units), piv)
    cost = lifetime[keep, None] * dist[keep]
    cap = allocator.budget_cap(nominal_bits, keep.size)
    if mode == 0:
        alloc = allocator.dp_allocate_budget(cost, bits, cap)
    else:
        alloc = allocator.lagrangian_allocate(cost, bits, cap)
    widths = np.full(n_units, PIVOT_BITS, dtype=np.uint8)
    widths[keep] = alloc.astype(np.uint8)
    return dict(mode=mode, n_layers=n_layers, n_heads=n_heads, d=D, n_pivots=n_pivots,
                bitset=bits, nominal_bits=nominal_bits, horizon=horizon, widths=widths,
                wbar=np.asarray(stats["wbar"], np.float32).reshape(-1),
                rho=np.asarray(stats["rho"], np.float32).reshape(-1),
                lgate=lgate, lifetime=np.asarray(lifetime, np.float64), scale_bits=int(scale_bits))


def uniform_plan(mode: int, D: int, n_layers: int, n_heads: int, bits: int, quantizer: int,
                 horizon: int, wbar=None, scale_bits: int = 32) -> dict:
    """A baseline plan: every unit at `bits`, no pivots (实验: uniform INT-b).
    wbar defaults to ones (rho = 1); lgate is 0, so L_u = horizon."""
    n_units = n_layers * n_heads * (D if mode == 1 else 1)
    nrow = n_layers * n_heads * D
    wbar = np.ones(nrow, np.float32) if wbar is None else np.asarray(wbar, np.float32).reshape(-1)
    rho = np.array([1.0 / math.sqrt(math.sqrt(float(x))) for x in wbar], dtype=np.float32)
    return dict(mode=mode, n_layers=n_layers, n_heads=n_heads, d=D, n_pivots=0, bitset=[int(bits)],
                nominal_bits=float(bits), horizon=horizon, widths=np.full(n_units, int(bits), np.uint8),
                wbar=wbar, rho=rho, lgate=np.zeros(n_units), lifetime=np.full(n_units, float(horizon)),
                quantizer=int(quantizer), scale_bits=int(scale_bits))


def slice_plan(plan: dict, lb: int, le: int) -> dict:
    """The plan of layers [lb, le): their units and row weights, the parent's
    other fields; n_pivots counts the slice's FP16 units; nominal bits are the
    slice's own average width, the smallest float32 whose floor(nominal * N)
    covers the widths (a global budget is not a per-layer constraint)."""
    L, H, D = int(plan["n_layers"]), int(plan["n_heads"]), int(plan["d"])
    per_units = H if int(plan["mode"]) == 0 else H * D
    u = slice(lb * per_units, le * per_units)
    rows = slice(lb * H * D, le * H * D)
    widths = np.asarray(plan["widths"], np.uint8)[u].copy()
    q = widths[widths != PIVOT_BITS].astype(np.int64)
    nominal = np.float32(plan["nominal_bits"])
    if q.size:
        nominal = np.float32(int(q.sum()) / q.size)
        while math.floor(float(nominal) * q.size) < int(q.sum()):
            nominal = np.nextafter(nominal, np.float32(1e30))
    out = dict(plan)
    out.update(n_layers=le - lb, widths=widths, n_pivots=int((widths == PIVOT_BITS).sum()),
               nominal_bits=float(nominal), wbar=np.asarray(plan["wbar"], np.float32).reshape(-1)[rows].copy(),
               rho=np.asarray(plan["rho"], np.float32).reshape(-1)[rows].copy(),
               lgate=np.asarray(plan["lgate"], np.float64)[u].copy(),
               lifetime=np.asarray(plan["lifetime"], np.float64)[u].copy())
    return out


def lifetime_l_from_halflife(h: float) -> float:
    return -math.log(2.0) / h
