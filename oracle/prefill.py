"""Chunked prefill of one per-head state -- CPU oracle, TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg use it.

The step before decode: a prompt of T tokens runs the same gated delta rule
as the decode step (STEPQuant paper digest page, 背景与动机; the recurrence
reading with the gate applied first),

    S_t = (I - beta_t k_t k_t^T) alpha_t S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t,

with a scalar retention gate alpha_t per (token, head).  Writing
u_t = v_t - alpha_t S_{t-1}^T k_t, the step is S_t = alpha_t S_{t-1} +
beta_t k_t u_t^T.  Unrolled over a chunk of C tokens that starts from S_0,
with gamma_t = alpha_1 ... alpha_t and Gamma_ts = gamma_t / gamma_s:

    (I + M) U = V - diag(gamma) K S_0,   M_ts = Gamma_ts beta_s (k_t . k_s) for s < t
    O   = diag(gamma) Q S_0 + (L_incl(Q K^T o Gamma) diag(beta)) U
    S_C = gamma_C S_0 + K^T diag(beta gamma_C / gamma) U

(rows of K, V, Q, U, O are tokens; L_incl keeps s <= t).  The chunk form does
the same arithmetic in dense products, which is what lets a prefill run on
matrix units; this module evaluates it in fp64 as written and is pinned
against the sequential fp64 recurrence.

Per-key-row units (KDA: a gate alpha_t in R^D per token, applied first as
Diag(alpha_t), the order of the recurrence reading for per-row gates): with
u_t = v_t - S_{t-1}^T Diag(alpha_t) k_t the step is S_t = Diag(alpha_t) S_{t-1}
+ beta_t k_t u_t^T, and with Gamma_t = alpha_1 o ... o alpha_t per key row,

    (I + M) U = V - (K o Gamma) S_0,   M_ts = beta_s sum_i k_ti k_si Gamma_ti / Gamma_si  (s < t)
    O   = (Q o Gamma) S_0 + L_incl(A) U,  A_ts = beta_s sum_i q_ti k_si Gamma_ti / Gamma_si
    S_C = Diag(Gamma_C) S_0 + (K o (Gamma_C / Gamma) o beta)^T U
"""
from __future__ import annotations

import numpy as np

from . import core


def sequential(S0, Q, K, V, alpha, beta):
    """The recurrence token by token in fp64 (core.step_fp64).
    S0 [D, D]; Q, K, V [T, D]; alpha, beta [T].  Returns (O [T, D], S_T)."""
    S = np.array(S0, dtype=np.float64, order="C", copy=True)
    O = np.zeros((len(alpha), S.shape[1]))
    for t in range(len(alpha)):
        O[t] = core.step_fp64(S, Q[t], K[t], V[t], alpha[t], beta[t])
    return O, S


def chunk(S0, Q, K, V, alpha, beta):
    """One chunk of the formulas above in fp64.  Returns (O, S_C)."""
    S0 = np.asarray(S0, np.float64)
    Q, K, V = (np.asarray(x, np.float64) for x in (Q, K, V))
    a = np.asarray(alpha, np.float64)
    b = np.asarray(beta, np.float64)
    C = len(a)
    gamma = np.cumprod(a)
    ratio = gamma[:, None] / gamma[None, :]                  # Gamma_ts
    strict = np.tril(np.ones((C, C), dtype=bool), -1)
    incl = np.tril(np.ones((C, C), dtype=bool), 0)
    M = np.where(strict, (K @ K.T) * ratio * b[None, :], 0.0)
    rhs = V - gamma[:, None] * (K @ S0)
    U = np.zeros_like(rhs)
    for t in range(C):                                       # forward substitution, (I + M) unit lower
        U[t] = rhs[t] - M[t, :t] @ U[:t]
    A = np.where(incl, (Q @ K.T) * ratio * b[None, :], 0.0)
    O = gamma[:, None] * (Q @ S0) + A @ U
    S = gamma[-1] * S0 + K.T @ ((b * gamma[-1] / gamma)[:, None] * U)
    return O, S


def chunked(S0, Q, K, V, alpha, beta, C=64):
    """A whole prompt in chunks of C tokens (the last one ragged).
    Returns (O [T, D], S_T)."""
    T = len(alpha)
    S = np.asarray(S0, np.float64)
    O = np.zeros((T, S.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        O[c0:c1], S = chunk(S, Q[c0:c1], K[c0:c1], V[c0:c1], alpha[c0:c1], beta[c0:c1])
    return O, S


def chunk_rows(S0, Q, K, V, alpha, beta):
    """One chunk of the per-key-row formulas above in fp64; alpha [C, D].
    The ratios Gamma_ti / Gamma_si are formed per (t, s, i) as written.
    Returns (O, S_C)."""
    S0 = np.asarray(S0, np.float64)
    Q, K, V = (np.asarray(x, np.float64) for x in (Q, K, V))
    a = np.asarray(alpha, np.float64)
    b = np.asarray(beta, np.float64)
    C = len(b)
    gamma = np.cumprod(a, axis=0)                            # [C, D]
    ratio = gamma[:, None, :] / gamma[None, :, :]            # [t, s, i]
    strict = np.tril(np.ones((C, C), dtype=bool), -1)
    incl = np.tril(np.ones((C, C), dtype=bool), 0)
    M = np.where(strict, np.einsum("ti,si,tsi->ts", K, K, ratio) * b[None, :], 0.0)
    rhs = V - (K * gamma) @ S0
    U = np.zeros_like(rhs)
    for t in range(C):                                       # forward substitution, (I + M) unit lower
        U[t] = rhs[t] - M[t, :t] @ U[:t]
    A = np.where(incl, np.einsum("ti,si,tsi->ts", Q, K, ratio) * b[None, :], 0.0)
    O = (Q * gamma) @ S0 + A @ U
    S = gamma[-1][:, None] * S0 + (K * (gamma[-1][None, :] / gamma) * b[:, None]).T @ U
    return O, S


def chunked_rows(S0, Q, K, V, alpha, beta, C=64):
    """A whole prompt with per-key-row gates (alpha [T, D]) in chunks of C tokens."""
    T = len(beta)
    S = np.asarray(S0, np.float64)
    O = np.zeros((T, S.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        O[c0:c1], S = chunk_rows(S, Q[c0:c1], K[c0:c1], V[c0:c1], alpha[c0:c1], beta[c0:c1])
    return O, S
