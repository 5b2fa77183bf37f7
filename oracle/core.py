"""ctypes bindings of the C oracle (stepq_oracle.c) -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may
import this module.  It never loads the product library and the product never
loads it.

Source of every formula: the STEPQuant paper digest page (vibe-research),
sections 背景与动机, 方法-1 .. 方法-4; readings are stated in stepq_oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "stepq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libstepq_oracle.so")

PIVOT_BITS = 16

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with no floating-point contraction and no fast-math."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


P = ctypes.c_void_p
I = ctypes.c_int
L = ctypes.c_long
F = ctypes.c_float
D = ctypes.c_double


def _declare(l):
    l.sq_f16_to_f32.argtypes = [ctypes.c_uint16]
    l.sq_f16_to_f32.restype = F
    l.sq_f32_to_f16.argtypes = [F]
    l.sq_f32_to_f16.restype = ctypes.c_uint16
    l.sq_codes_bytes_uniform.argtypes = [I, I]
    l.sq_codes_bytes_uniform.restype = L
    l.sq_pack_uniform.argtypes = [I, I, P, P]
    l.sq_unpack_uniform.argtypes = [I, I, P, P]
    l.sq_row_bytes.argtypes = [I, I]
    l.sq_row_bytes.restype = L
    l.sq_codes_bytes_rows.argtypes = [I, P]
    l.sq_codes_bytes_rows.restype = L
    l.sq_pack_rows.argtypes = [I, P, P, P, P]
    l.sq_unpack_rows.argtypes = [I, P, P, P, P]
    l.sq_codes_bytes_bands.argtypes = [I, P]
    l.sq_codes_bytes_bands.restype = L
    l.sq_pack_bands.argtypes = [I, P, P, P, P]
    l.sq_unpack_bands.argtypes = [I, P, P, P, P]
    l.sq_pairwise_sum.argtypes = [P, I]
    l.sq_pairwise_sum.restype = F
    l.sq_band_dot.argtypes = [I, P, I, P, I]
    l.sq_band_dot.restype = F
    l.sq_quantize.argtypes = [I, P, P, P, P, P, P, P, P, P, P]
    l.sq_quantize_absmax.argtypes = [I, P, P, P, P, P, P, P]
    l.sq_quantize_s.argtypes = [I, P, P, P, P, P, P, P, P, P, P, I]
    l.sq_quantize_absmax_s.argtypes = [I, P, P, P, P, P, P, P, I]
    l.sq_f32_to_bf16.argtypes = [F]
    l.sq_f32_to_bf16.restype = ctypes.c_uint16
    l.sq_bf16_to_f32.argtypes = [ctypes.c_uint16]
    l.sq_bf16_to_f32.restype = F
    l.sq_reconstruct.argtypes = [I, P, P, P, P, P, P]
    l.sq_step_from_codes.argtypes = [I, P, P, P, P, P, P, P, P, P, F, P, P, P, P]
    l.sq_step_fp32.argtypes = [I, P, P, P, P, P, F, P]
    l.sq_step_fp64.argtypes = [I, P, P, P, P, P, D, P]
    l.sq_calib_accumulate.argtypes = [I, P, P, P, F, P, P]
    l.sq_distortion_rows.argtypes = [I, I, P, P, P, P]
    l.sq_lifetime_weight.argtypes = [D, L]
    l.sq_lifetime_weight.restype = D


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


# --------------------------------------------------------------------------
# binary16
# --------------------------------------------------------------------------

def f16_to_f32(bits: int) -> float:
    return float(lib().sq_f16_to_f32(int(bits)))


def f32_to_f16(x: float) -> int:
    return int(lib().sq_f32_to_f16(float(np.float32(x))))


# --------------------------------------------------------------------------
# packed format
# --------------------------------------------------------------------------

def codes_bytes_uniform(D: int, b: int) -> int:
    return int(lib().sq_codes_bytes_uniform(D, b))


def pack_uniform(D: int, b: int, z: np.ndarray) -> np.ndarray:
    z = _i32(z).reshape(D, D)
    out = np.zeros(codes_bytes_uniform(D, b), dtype=np.uint8)
    lib().sq_pack_uniform(D, b, _p(z), _p(out))
    return out


def unpack_uniform(D: int, b: int, blk: np.ndarray) -> np.ndarray:
    blk = np.ascontiguousarray(blk, dtype=np.uint8)
    z = np.zeros((D, D), dtype=np.int32)
    lib().sq_unpack_uniform(D, b, _p(blk), _p(z))
    return z


def codes_bytes_rows(D: int, widths) -> int:
    w = _i32(widths)
    return int(lib().sq_codes_bytes_rows(D, _p(w)))


def pack_rows(D: int, widths, z: np.ndarray, h: np.ndarray) -> np.ndarray:
    w = _i32(widths)
    z = _i32(z).reshape(D, D)
    h = np.ascontiguousarray(h, dtype=np.uint16).reshape(D, D)
    out = np.zeros(codes_bytes_rows(D, w), dtype=np.uint8)
    lib().sq_pack_rows(D, _p(w), _p(z), _p(h), _p(out))
    return out


def unpack_rows(D: int, widths, blk: np.ndarray):
    w = _i32(widths)
    blk = np.ascontiguousarray(blk, dtype=np.uint8)
    z = np.zeros((D, D), dtype=np.int32)
    h = np.zeros((D, D), dtype=np.uint16)
    lib().sq_unpack_rows(D, _p(w), _p(blk), _p(z), _p(h))
    return z, h


def codes_bytes_bands(D: int, widths) -> int:
    w = _i32(widths)
    return int(lib().sq_codes_bytes_bands(D, _p(w)))


def pack_bands(D: int, widths, z: np.ndarray, h: np.ndarray) -> np.ndarray:
    w = _i32(widths)
    z = _i32(z).reshape(D, D)
    h = np.ascontiguousarray(h, dtype=np.uint16).reshape(D, D)
    out = np.zeros(codes_bytes_bands(D, w), dtype=np.uint8)
    lib().sq_pack_bands(D, _p(w), _p(z), _p(h), _p(out))
    return out


def unpack_bands(D: int, widths, blk: np.ndarray):
    w = _i32(widths)
    blk = np.ascontiguousarray(blk, dtype=np.uint8)
    z = np.zeros((D, D), dtype=np.int32)
    h = np.zeros((D, D), dtype=np.uint16)
    lib().sq_unpack_bands(D, _p(w), _p(blk), _p(z), _p(h))
    return z, h


# --------------------------------------------------------------------------
# arithmetic
# --------------------------------------------------------------------------

def pairwise_sum(x: np.ndarray) -> np.float32:
    x = _f32(x)
    return np.float32(lib().sq_pairwise_sum(_p(x), x.size))


def band_dot(x: np.ndarray, y: np.ndarray) -> np.float32:
    """sum_i x_i y_i over D = len(x) rows in band order (see sq_band_dot)."""
    x = _f32(x)
    y = _f32(y)
    assert x.size == y.size and x.size % 16 == 0
    return np.float32(lib().sq_band_dot(x.size, _p(x), 1, _p(y), 1))


def f32_to_bf16(x: float) -> int:
    return int(lib().sq_f32_to_bf16(float(x)))


def bf16_to_f32(bits: int) -> float:
    return float(lib().sq_bf16_to_f32(int(bits)))


def quantize(D: int, widths, rho, wbar, S, return_z0: bool = False, scale_bits: int = 32):
    """Return (z, h, r, c, tie[, z0]) for one head (see sq_quantize_s)."""
    w = _i32(widths)
    rho = _f32(rho)
    wbar = _f32(wbar)
    S = _f32(S).reshape(D, D)
    z = np.zeros((D, D), dtype=np.int32)
    h = np.zeros((D, D), dtype=np.uint16)
    r = np.zeros(D, dtype=np.float32)
    c = np.zeros(D, dtype=np.float32)
    tie = np.zeros((D, D), dtype=np.uint8)
    z0 = np.zeros((D, D), dtype=np.int32)
    lib().sq_quantize_s(D, _p(w), _p(rho), _p(wbar), _p(S), _p(z), _p(h), _p(r), _p(c), _p(tie), _p(z0),
                        int(scale_bits))
    if return_z0:
        return z, h, r, c, tie, z0
    return z, h, r, c, tie


def quantize_absmax(D: int, widths, S, scale_bits: int = 32):
    """Return (z, h, r, c, tie) for one head under the per-row absmax
    quantizer (see sq_quantize_absmax)."""
    w = _i32(widths)
    S = _f32(S).reshape(D, D)
    z = np.zeros((D, D), dtype=np.int32)
    h = np.zeros((D, D), dtype=np.uint16)
    r = np.zeros(D, dtype=np.float32)
    c = np.zeros(D, dtype=np.float32)
    tie = np.zeros((D, D), dtype=np.uint8)
    lib().sq_quantize_absmax_s(D, _p(w), _p(S), _p(z), _p(h), _p(r), _p(c), _p(tie), int(scale_bits))
    return z, h, r, c, tie


def reconstruct(D: int, widths, z, h, r, c) -> np.ndarray:
    w = _i32(widths)
    z = _i32(z).reshape(D, D)
    h = np.ascontiguousarray(h, dtype=np.uint16).reshape(D, D)
    r = _f32(r)
    c = _f32(c)
    out = np.zeros((D, D), dtype=np.float32)
    lib().sq_reconstruct(D, _p(w), _p(z), _p(h), _p(r), _p(c), _p(out))
    return out


def step_from_codes(D: int, widths, z, h, r, c, q, k, v, alpha, beta):
    """One decode step from a head's stored (z, h, r, c).

    alpha: scalar (GDN) or D values (KDA).  Returns (S_t fp32, o, u, w)."""
    w = _i32(widths)
    z = _i32(z).reshape(D, D)
    h = np.ascontiguousarray(h, dtype=np.uint16).reshape(D, D)
    al = np.broadcast_to(np.asarray(alpha, dtype=np.float32), (D,)).copy()
    S = np.zeros((D, D), dtype=np.float32)
    o = np.zeros(D, dtype=np.float32)
    u = np.zeros(D, dtype=np.float32)
    ww = np.zeros(D, dtype=np.float32)
    lib().sq_step_from_codes(D, _p(w), _p(z), _p(h), _p(_f32(r)), _p(_f32(c)),
                             _p(_f32(q)), _p(_f32(k)), _p(_f32(v)), _p(al),
                             float(np.float32(beta)), _p(S), _p(o), _p(u), _p(ww))
    return S, o, u, ww


def step_fp32(S: np.ndarray, q, k, v, alpha, beta):
    """In-place fp32 recurrence step; returns o."""
    D = S.shape[0]
    assert S.dtype == np.float32 and S.flags["C_CONTIGUOUS"]
    al = np.broadcast_to(np.asarray(alpha, dtype=np.float32), (D,)).copy()
    o = np.zeros(D, dtype=np.float32)
    lib().sq_step_fp32(D, _p(S), _p(_f32(q)), _p(_f32(k)), _p(_f32(v)), _p(al),
                       float(np.float32(beta)), _p(o))
    return o


def step_fp64(S: np.ndarray, q, k, v, alpha, beta):
    """In-place fp64 recurrence step; returns o."""
    D = S.shape[0]
    assert S.dtype == np.float64 and S.flags["C_CONTIGUOUS"]
    f = lambda a: np.ascontiguousarray(a, dtype=np.float64)
    al = np.broadcast_to(np.asarray(alpha, dtype=np.float64), (D,)).copy()
    o = np.zeros(D, dtype=np.float64)
    lib().sq_step_fp64(D, _p(S), _p(f(q)), _p(f(k)), _p(f(v)), _p(al), float(beta), _p(o))
    return o


def calib_accumulate(q, k, alpha, beta, omega_acc: np.ndarray, lsum_acc: np.ndarray):
    D = omega_acc.shape[0]
    al = np.broadcast_to(np.asarray(alpha, dtype=np.float32), (D,)).copy()
    lib().sq_calib_accumulate(D, _p(_f32(q)), _p(_f32(k)), _p(al), float(np.float32(beta)),
                              _p(omega_acc), _p(lsum_acc))


def distortion_rows(D: int, b: int, rho, wbar, S) -> np.ndarray:
    out = np.zeros(D, dtype=np.float64)
    lib().sq_distortion_rows(D, b, _p(_f32(rho)), _p(_f32(wbar)), _p(_f32(S).reshape(D, D)), _p(out))
    return out


def lifetime_weight(l: float, H: int) -> float:
    return float(lib().sq_lifetime_weight(float(l), int(H)))
