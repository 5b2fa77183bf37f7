"""Thin ctypes binding of libstepq.so (include/stepq.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libstepq.so.  PyTorch supplies device memory and streams.  There
is no fallback: if the library is missing or no sm_100 device is present,
the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstepq.so")

OK, EINVAL, EFORMAT, ECUDA, ETIMEDOUT, EDEVICE, ENOMEM = 0, -1, -2, -3, -4, -5, -6
PIVOT_BITS = 16

EXPORTED = [
    "stepq_plan_load", "stepq_plan_load_mem", "stepq_plan_free", "stepq_plan_get_info",
    "stepq_plan_widths", "stepq_plan_record", "stepq_plan_build", "stepq_ctx_create",
    "stepq_ctx_free", "stepq_workspace_bytes", "stepq_requant_pack", "stepq_decode_step",
    "stepq_decode_step_fused", "stepq_sync", "stepq_unpack", "stepq_fp32_decode_step",
    "stepq_calib_accumulate", "stepq_calib_distortion", "stepq_copy_probe",
    "stepq_launch_count", "stepq_last_error", "stepq_ctx_set_timing", "stepq_kernel_stats",
    "stepq_decode_step_noalloc", "stepq_plan_build_uniform", "stepq_ctx_set_wait_limit", "stepq_plan_slice", "stepq_prefill_fp32", "stepq_prefill",
    "stepq_prefill_workspace_bytes", "stepq_selftest_tc", "stepq_ctx_set_prefill_kernel",
    "stepq_ctx_set_step_kernel",
]
STEP_REGISTERS = 0    # fused step kernel: state in registers
STEP_TMEM = 1         # fused step kernel: state in tensor memory (per-head plans, d = 128)
PREFILL_MMA_SYNC = 0   # prefill kernel: mma.sync tiles, state in shared memory
PREFILL_TCGEN05 = 1    # prefill kernel: state in tensor memory, state products on tcgen05 (default)
QUANT_DUAL_AXIS = 0  # plan requantizer: STEPQuant row/column fit
QUANT_ABSMAX = 1     # plan requantizer: per-row absmax baseline, c = 1
NOALLOC_SCRATCH_BYTES = 8 << 20


class StepqError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"stepq error {code}: {msg}")
        self.code = code


class PlanInfo(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int), ("n_layers", ctypes.c_int), ("n_heads", ctypes.c_int),
        ("d", ctypes.c_int), ("n_units", ctypes.c_int), ("n_pivots", ctypes.c_int),
        ("bitset", ctypes.c_uint32), ("nominal_bits", ctypes.c_float), ("horizon", ctypes.c_uint64),
        ("slot_bytes", ctypes.c_uint64), ("bits_per_value", ctypes.c_double),
        ("bits_per_value_s16", ctypes.c_double), ("units_by_width", ctypes.c_int * 17),
        ("quantizer", ctypes.c_int), ("scale_bits", ctypes.c_int),
    ]


_lib = None
P = ctypes.c_void_p
I = ctypes.c_int


def lib():
    """Load libstepq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m quantized_recurrent_state_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        l.stepq_last_error.restype = ctypes.c_char_p
        l.stepq_plan_load.argtypes = [ctypes.c_char_p, ctypes.POINTER(P)]
        l.stepq_plan_load_mem.argtypes = [P, ctypes.c_size_t, ctypes.POINTER(P)]
        l.stepq_plan_free.argtypes = [P]
        l.stepq_plan_free.restype = None
        l.stepq_plan_get_info.argtypes = [P, ctypes.POINTER(PlanInfo)]
        l.stepq_plan_widths.argtypes = [P, P]
        l.stepq_plan_record.argtypes = [P, I, I, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64)]
        l.stepq_plan_build.argtypes = [I, I, I, I, P, I, ctypes.c_float, I, ctypes.c_uint64, P, P, P, I,
                                       ctypes.c_char_p, ctypes.POINTER(P)]
        l.stepq_plan_build_uniform.argtypes = [I, I, I, I, I, I, ctypes.c_uint64, P, I, ctypes.c_char_p,
                                               ctypes.POINTER(P)]
        l.stepq_plan_slice.argtypes = [P, I, I, ctypes.POINTER(P)]
        l.stepq_prefill_fp32.argtypes = [P, P, I, I, I, I, P, P, P, P, P, P, I]
        l.stepq_prefill.argtypes = [P, P, P, I, I, I, I, P, P, P, P, P, P, P, I]
        l.stepq_selftest_tc.argtypes = [P] * 6
        l.stepq_ctx_set_prefill_kernel.argtypes = [P, I]
        l.stepq_ctx_set_step_kernel.argtypes = [P, I]
        l.stepq_prefill_workspace_bytes.argtypes = [P, I, I]
        l.stepq_prefill_workspace_bytes.restype = ctypes.c_size_t
        l.stepq_ctx_create.argtypes = [P, P, P, I, I, ctypes.POINTER(P)]
        l.stepq_ctx_free.argtypes = [P]
        l.stepq_ctx_free.restype = None
        l.stepq_workspace_bytes.argtypes = [P, I, I]
        l.stepq_workspace_bytes.restype = ctypes.c_size_t
        l.stepq_requant_pack.argtypes = [P, P, P, I, I, I, P]
        l.stepq_decode_step.argtypes = [P, P, P, I, I, I, P, P, P, P, P, P, P]
        l.stepq_decode_step_fused.argtypes = [P, P, P, I, I, I, P, P, P, P, P, P]
        l.stepq_sync.argtypes = [P, I]
        l.stepq_unpack.argtypes = [P, P, P, I, I, I, P]
        l.stepq_fp32_decode_step.argtypes = [P, P, P, I, I, I, P, P, P, P, P, P]
        l.stepq_calib_accumulate.argtypes = [P, I, I, I, P, P, P, P, P, P]
        l.stepq_calib_distortion.argtypes = [P, I, I, I, P, P, P, I, P]
        l.stepq_copy_probe.argtypes = [P, P, ctypes.c_size_t, P]
        l.stepq_launch_count.argtypes = [P]
        l.stepq_launch_count.restype = ctypes.c_uint64
        l.stepq_ctx_set_timing.argtypes = [P, I]
        l.stepq_ctx_set_wait_limit.argtypes = [P, ctypes.c_uint32, ctypes.c_uint32]
        l.stepq_kernel_stats.argtypes = [P, P, P]
        l.stepq_decode_step_noalloc.argtypes = [P, P, P, I, I, I, P, P, P, P, P, P]
        _lib = l
    return _lib


def _check(rc: int):
    if rc != OK:
        raise StepqError(rc, lib().stepq_last_error().decode())
    return rc


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


class Plan:
    """A parsed, validated plan (host side)."""

    def __init__(self, handle):
        self._h = handle
        info = PlanInfo()
        _check(lib().stepq_plan_get_info(self._h, ctypes.byref(info)))
        self.info = info
        self.mode, self.n_layers, self.n_heads, self.d = info.mode, info.n_layers, info.n_heads, info.d
        self.slot_bytes = int(info.slot_bytes)

    @classmethod
    def load(cls, path: str) -> "Plan":
        h = P()
        _check(lib().stepq_plan_load(path.encode(), ctypes.byref(h)))
        return cls(h)

    @classmethod
    def from_bytes(cls, data: bytes) -> "Plan":
        h = P()
        buf = ctypes.create_string_buffer(data, len(data))
        _check(lib().stepq_plan_load_mem(buf, len(data), ctypes.byref(h)))
        return cls(h)

    @classmethod
    def build(cls, mode, n_layers, n_heads, d, bits, nominal_bits, n_pivots, horizon,
              lgate, dist, wbar, path=None, scale_bits=32) -> "Plan":
        bits_a = np.ascontiguousarray(bits, dtype=np.int32)
        lg = np.ascontiguousarray(lgate, dtype=np.float64)
        di = np.ascontiguousarray(dist, dtype=np.float64)
        wb = np.ascontiguousarray(wbar, dtype=np.float32)
        h = P()
        _check(lib().stepq_plan_build(mode, n_layers, n_heads, d, bits_a.ctypes.data, len(bits_a),
                                      float(nominal_bits), n_pivots, int(horizon), lg.ctypes.data,
                                      di.ctypes.data, wb.ctypes.data, int(scale_bits),
                                      path.encode() if path else None, ctypes.byref(h)))
        return cls(h)

    @classmethod
    def build_uniform(cls, mode, n_layers, n_heads, d, bits, quantizer=QUANT_DUAL_AXIS, horizon=65536,
                      wbar=None, path=None, scale_bits=32) -> "Plan":
        wb = None if wbar is None else np.ascontiguousarray(wbar, dtype=np.float32)
        h = P()
        _check(lib().stepq_plan_build_uniform(mode, n_layers, n_heads, d, int(bits), int(quantizer), int(horizon),
                                              None if wb is None else wb.ctypes.data, int(scale_bits),
                                              path.encode() if path else None, ctypes.byref(h)))
        return cls(h)

    def slice(self, lb: int, le: int) -> "Plan":
        """The plan of layers [lb, le) (its own pool layout)."""
        h = P()
        _check(lib().stepq_plan_slice(self._h, int(lb), int(le), ctypes.byref(h)))
        return Plan(h)

    def widths(self) -> np.ndarray:
        out = np.zeros(self.info.n_units, dtype=np.uint8)
        _check(lib().stepq_plan_widths(self._h, out.ctypes.data))
        return out

    def record(self, layer: int, head: int):
        off, nb = ctypes.c_uint64(), ctypes.c_uint64()
        _check(lib().stepq_plan_record(self._h, layer, head, ctypes.byref(off), ctypes.byref(nb)))
        return int(off.value), int(nb.value)

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.stepq_plan_free(self._h)
            self._h = None


class Context:
    """A plan bound to the current CUDA device with a main and a side stream."""

    def __init__(self, plan: Plan, n_slots: int, main_stream=None, side_stream=None, chunk_layers: int = 4):
        import torch
        self.plan = plan
        self.main = main_stream if main_stream is not None else torch.cuda.Stream()
        self.side = side_stream if side_stream is not None else torch.cuda.Stream()
        h = P()
        _check(lib().stepq_ctx_create(plan._h, ctypes.c_void_p(self.main.cuda_stream),
                                      ctypes.c_void_p(self.side.cuda_stream), n_slots, chunk_layers,
                                      ctypes.byref(h)))
        self._h = h
        self.n_slots = n_slots

    def _after_caller(self):
        """Order the context's main stream after the caller's current torch
        stream, so that tensors produced there are complete before the
        library's kernels read or write them."""
        import torch
        cur = torch.cuda.current_stream()
        if cur.cuda_stream != self.main.cuda_stream:
            self.main.wait_stream(cur)

    def workspace_bytes(self, n_req: int, n_layers: int) -> int:
        return int(lib().stepq_workspace_bytes(self._h, n_req, n_layers))

    def requant_pack(self, pool, slots, n_req, lb, le, S):
        self._after_caller()
        return _check(lib().stepq_requant_pack(self._h, _ptr(pool), _ptr(slots), n_req, lb, le, _ptr(S)))

    def decode_step(self, pool, slots, n_req, lb, le, q, k, v, alpha, beta, o, workspace):
        self._after_caller()
        return _check(lib().stepq_decode_step(self._h, _ptr(pool), _ptr(slots), n_req, lb, le, _ptr(q),
                                              _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
                                              _ptr(workspace)))

    def decode_step_fused(self, pool, slots, n_req, lb, le, q, k, v, alpha, beta, o):
        self._after_caller()
        return _check(lib().stepq_decode_step_fused(self._h, _ptr(pool), _ptr(slots), n_req, lb, le,
                                                    _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                                    _ptr(o)))

    def decode_step_noalloc(self, pool, slots, n_req, lb, le, q, k, v, alpha, beta, o):
        """The two-stream step without a workspace argument: for callers that
        cannot allocate device memory.  The hand-off values live in a fixed
        8 MiB array inside the library (shared by all calls on the device)."""
        self._after_caller()
        return _check(lib().stepq_decode_step_noalloc(self._h, _ptr(pool), _ptr(slots), n_req, lb, le,
                                                      _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                                      _ptr(o)))

    def sync(self, timeout_ms: int = 60000):
        return _check(lib().stepq_sync(self._h, timeout_ms))

    def unpack(self, pool, slots, n_req, lb, le, S):
        self._after_caller()
        return _check(lib().stepq_unpack(self._h, _ptr(pool), _ptr(slots), n_req, lb, le, _ptr(S)))

    def fp32_decode_step(self, S_pool, slots, n_req, lb, le, q, k, v, alpha, beta, o):
        self._after_caller()
        return _check(lib().stepq_fp32_decode_step(self._h, _ptr(S_pool), _ptr(slots), n_req, lb, le,
                                                   _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                                   _ptr(o)))

    def prefill_fp32(self, S, n_req, lb, le, T, q, k, v, alpha, beta, o, zero_init=False):
        self._after_caller()
        return _check(lib().stepq_prefill_fp32(self._h, _ptr(S), n_req, lb, le, int(T), _ptr(q), _ptr(k), _ptr(v),
                                               _ptr(alpha), _ptr(beta), _ptr(o), 1 if zero_init else 0))

    def set_step_kernel(self, kernel: int):
        return _check(lib().stepq_ctx_set_step_kernel(self._h, kernel))

    def set_prefill_kernel(self, kernel: int):
        return _check(lib().stepq_ctx_set_prefill_kernel(self._h, kernel))

    def prefill_workspace_bytes(self, n_req: int, n_layers: int) -> int:
        return int(lib().stepq_prefill_workspace_bytes(self._h, n_req, n_layers))

    def prefill(self, pool, slots, n_req, lb, le, T, q, k, v, alpha, beta, o, workspace, from_zero=False):
        self._after_caller()
        return _check(lib().stepq_prefill(self._h, _ptr(pool), _ptr(slots), n_req, lb, le, int(T), _ptr(q), _ptr(k),
                                          _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o), _ptr(workspace),
                                          1 if from_zero else 0))

    def calib_accumulate(self, n_req, lb, le, q, k, alpha, beta, omega_acc, lsum_acc):
        self._after_caller()
        return _check(lib().stepq_calib_accumulate(self._h, n_req, lb, le, _ptr(q), _ptr(k), _ptr(alpha),
                                                   _ptr(beta), _ptr(omega_acc), _ptr(lsum_acc)))

    def calib_distortion(self, n_req, lb, le, S, wbar, bits, dist_acc):
        self._after_caller()
        b = (ctypes.c_int * len(bits))(*[int(x) for x in bits])
        return _check(lib().stepq_calib_distortion(self._h, n_req, lb, le, _ptr(S), _ptr(wbar), b,
                                                   len(bits), _ptr(dist_acc)))

    def set_timing(self, on: bool):
        return _check(lib().stepq_ctx_set_timing(self._h, 1 if on else 0))

    def set_wait_limit(self, polls: int = 0, phantom_bytes: int = 0):
        """Copy-wait poll limit of later launches (0: default); phantom_bytes > 0
        makes every wait run out (tests of the timeout path)."""
        return _check(lib().stepq_ctx_set_wait_limit(self._h, int(polls), int(phantom_bytes)))

    def kernel_stats(self):
        """{kind: (total ms, launches)} of the launches timed since the last call."""
        ms = (ctypes.c_double * 5)()
        n = (ctypes.c_uint64 * 5)()
        _check(lib().stepq_kernel_stats(self._h, ms, n))
        names = ("decode", "fitpack", "fused", "other", "prefill")
        return {names[i]: (float(ms[i]), int(n[i])) for i in range(5)}

    @property
    def launches(self) -> int:
        return int(lib().stepq_launch_count(self._h))

    def close(self):
        if getattr(self, "_h", None):
            lib().stepq_ctx_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def selftest_tc(A, B1, B2, D1, D2, D3):
    """stepq_selftest_tc: D1 = A B1^T, D2 = D1 B2^T, D3 = A B2^T on the tensor cores (device
    tensors: A [128][32], B1 [32][32], B2 [64][32], D1 [128][32], D2 and D3 [128][64])."""
    return _check(lib().stepq_selftest_tc(_ptr(A), _ptr(B1), _ptr(B2), _ptr(D1), _ptr(D2), _ptr(D3)))


def copy_probe(dst, src, nbytes: int, stream):
    return _check(lib().stepq_copy_probe(_ptr(dst), _ptr(src), nbytes, ctypes.c_void_p(stream.cuda_stream)))
