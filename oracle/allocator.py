"""Offline lifetime-aware bit allocation -- oracle side, TEST INFRASTRUCTURE.

Source: STEPQuant paper digest page (vibe-research), section
"方法-1 Lifetime-aware Bit Allocation": unit u (a GDN head or a KDA key row)
has distortion d_u(b) at b bits and mean log retention gate l_u; its error
lifetime weight over a horizon of H steps is L_u = sum_{j<H} exp(2 j l_u);
the plan minimises sum_u L_u d_u(b_u) under an average-bit budget, with
multiple-choice dynamic programming for per-head units and a Lagrangian
allocation with discrete budget repair for per-row units.  A fixed number
of the hardest units is kept in FP16 (pivots).

Readings (the pages give no formulas beyond the objective):
  * pivots are the top-P units by L_u * d_u(b_max), ties to the lower index;
  * the budget covers the non-pivot units: sum b_u <= floor(B_nom * N);
  * ties in the DP go to (cost, total bits, lexicographically smaller
    width vector); the Lagrangian takes, per unit, the width minimising
    L_u d_u(b) + lambda b (ties to the smaller width), bisects lambda in fp64
    for 200 iterations for the smallest feasible value, then upgrades, while
    at least 2 bits of slack remain, the unit with the largest cost drop per
    2 bits (ties to the lower index), stopping when no upgrade lowers cost.
"""
from __future__ import annotations

import itertools
import math

import numpy as np

PIVOT_BITS = 16


def lifetime_weight_closed_form(l: float, H: int) -> float:
    """(1 - e^{2Hl}) / (1 - e^{2l}) for l < 0; H at l = 0 (used by the pins)."""
    if l == 0.0:
        return float(H)
    return math.expm1(2.0 * H * l) / math.expm1(2.0 * l)


def select_pivots(L: np.ndarray, d_max: np.ndarray, n_pivots: int) -> np.ndarray:
    """Indices of the top-n_pivots units by L_u * d_u(b_max), ties to lower index."""
    score = np.asarray(L, dtype=np.float64) * np.asarray(d_max, dtype=np.float64)
    order = sorted(range(len(score)), key=lambda u: (-score[u], u))
    return np.array(sorted(order[:n_pivots]), dtype=np.int64)


def budget_cap(nominal_bits: float, n_units: int) -> int:
    return int(math.floor(float(nominal_bits) * n_units))


def dp_allocate_budget(cost: np.ndarray, widths, cap_bits: int) -> np.ndarray:
    """Multiple-choice DP.  cost[u, m] = L_u d_u(widths[m]); widths ascending
    even integers spaced by 2.  Returns the chosen width per unit with
    sum(width) <= cap_bits."""
    cost = np.asarray(cost, dtype=np.float64)
    widths = list(widths)
    N, M = cost.shape
    bmin = widths[0]
    steps = [(w - bmin) // 2 for w in widths]
    C = (cap_bits - bmin * N) // 2
    if C < 0:
        raise ValueError("budget below the minimum width")
    C = min(C, steps[-1] * N)
    INF = np.inf
    # V[u] over capacity c (at most c steps for units u..N-1): (cost, bits)
    Vc = np.zeros(C + 1)
    Vb = np.zeros(C + 1, dtype=np.int64)
    Vc_all = [None] * (N + 1)
    Vb_all = [None] * (N + 1)
    Vc_all[N], Vb_all[N] = Vc, Vb
    for u in range(N - 1, -1, -1):
        bestc = np.full(C + 1, INF)
        bestb = np.zeros(C + 1, dtype=np.int64)
        for m in range(M):
            s = steps[m]
            candc = np.full(C + 1, INF)
            candb = np.zeros(C + 1, dtype=np.int64)
            if s <= C:
                candc[s:] = cost[u, m] + Vc_all[u + 1][: C + 1 - s]
                candb[s:] = widths[m] + Vb_all[u + 1][: C + 1 - s]
            better = (candc < bestc) | ((candc == bestc) & (candb < bestb))
            bestc = np.where(better, candc, bestc)
            bestb = np.where(better, candb, bestb)
        Vc_all[u], Vb_all[u] = bestc, bestb
    # forward reconstruction: smallest width reaching the optimum at each unit
    out = np.zeros(N, dtype=np.int64)
    c = C
    for u in range(N):
        target = (Vc_all[u][c], Vb_all[u][c])
        for m in range(M):
            s = steps[m]
            if s > c:
                continue
            tc = cost[u, m] + Vc_all[u + 1][c - s]
            tb = widths[m] + Vb_all[u + 1][c - s]
            if tc == target[0] and tb == target[1]:
                out[u] = widths[m]
                c -= s
                break
        else:  # pragma: no cover - unreachable when the DP is consistent
            raise RuntimeError("DP reconstruction failed")
    return out


def _lagrange_choice(cost: np.ndarray, widths, lam: float) -> np.ndarray:
    w = np.asarray(widths, dtype=np.float64)
    obj = cost + lam * w[None, :]
    # argmin with ties to the smaller width: first index of the minimum
    return np.asarray(widths)[np.argmin(obj, axis=1)]


def lagrangian_allocate(cost: np.ndarray, widths, cap_bits: int, iters: int = 200) -> np.ndarray:
    cost = np.asarray(cost, dtype=np.float64)
    widths = list(widths)
    N = cost.shape[0]
    if widths[0] * N > cap_bits:
        raise ValueError("budget below the minimum width")
    b = _lagrange_choice(cost, widths, 0.0)
    if b.sum() > cap_bits:
        lo, hi = 0.0, 1.0
        while _lagrange_choice(cost, widths, hi).sum() > cap_bits:
            hi *= 2.0
        for _ in range(iters):
            mid = 0.5 * (lo + hi)
            if _lagrange_choice(cost, widths, mid).sum() <= cap_bits:
                hi = mid
            else:
                lo = mid
        b = _lagrange_choice(cost, widths, hi)
    # discrete repair
    idx = {w: m for m, w in enumerate(widths)}
    slack = cap_bits - int(b.sum())
    while slack >= 2:
        best_u, best_drop = -1, 0.0
        for u in range(N):
            m = idx[int(b[u])]
            if m + 1 >= len(widths):
                continue
            drop = cost[u, m] - cost[u, m + 1]
            if drop > best_drop:
                best_u, best_drop = u, drop
        if best_u < 0:
            break
        b[best_u] = widths[idx[int(b[best_u])] + 1]
        slack -= 2
    return b.astype(np.int64)


def total_cost(cost: np.ndarray, widths, alloc) -> float:
    """Sum over units, accumulated from the last unit to the first (the DP's order)."""
    idx = {w: m for m, w in enumerate(widths)}
    s = 0.0
    for u in range(len(alloc) - 1, -1, -1):
        s = cost[u, idx[int(alloc[u])]] + s
    return s


def brute_force(cost: np.ndarray, widths, cap_bits: int) -> np.ndarray:
    """Exhaustive search with the DP's tie rule (cost, bits, lexicographic)."""
    cost = np.asarray(cost, dtype=np.float64)
    N = cost.shape[0]
    best = None
    for combo in itertools.product(widths, repeat=N):  # lexicographic order
        bits = sum(combo)
        if bits > cap_bits:
            continue
        key = (total_cost(cost, widths, combo), bits)
        if best is None or key < best[0]:
            best = (key, combo)
    return np.array(best[1], dtype=np.int64)


def bits_per_value(mode: int, n_layers: int, n_heads: int, D: int, unit_widths,
                   scale_bits: int = 32) -> float:
    """Real bit/value including pivots and scale metadata ("方法-1": the
    compression ratios count the compact representation, not 32/b).

    Codes: b bits per value of a non-pivot unit, 16 per pivot value.  Scales:
    one row factor per non-pivot key row and one column factor per value
    column of every head that has a non-pivot row, scale_bits each."""
    w = np.asarray(unit_widths).astype(np.int64)
    n_heads_tot = n_layers * n_heads
    if mode == 0:
        assert w.size == n_heads_tot
        code_bits = float((w * D * D).sum())
        nonpiv = w != PIVOT_BITS
        scale = scale_bits * (D * nonpiv.sum() + D * nonpiv.sum())
    else:
        assert w.size == n_heads_tot * D
        code_bits = float((w * D).sum())
        rows = w.reshape(n_heads_tot, D)
        nonpiv_rows = (rows != PIVOT_BITS)
        scale = scale_bits * (nonpiv_rows.sum() + D * nonpiv_rows.any(axis=1).sum())
    values = n_heads_tot * D * D
    return (code_bits + float(scale)) / values
