"""Timestep-adaptive masked INT8 linear for NVIDIA B200 (sm_100a).

The compute path is libtasq.so (hand-written CUDA: a fused block-Hadamard + INT8 quantization
prologue and a tcgen05 INT8 GEMM that truncates weight bit planes in flight). This package is
its ctypes binding; see include/tasq.h for the C ABI.
"""
from .binding import *  # noqa: F401,F403
from .binding import LIB_PATH, Context, TasqError, lib  # noqa: F401
