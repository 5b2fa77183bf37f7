"""B200-native packed recurrent-state decode step (STEPQuant hot path).

The compute path lives in libstepq.so (CUDA for sm_100a, C ABI declared in
include/stepq.h).  `quantized_recurrent_state_b200.stepq` is the thin ctypes
binding; importing this package itself loads nothing.
"""
