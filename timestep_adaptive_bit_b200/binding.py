"""ctypes binding of libtasq (include/tasq.h): argument marshalling only.

Every function here has the name of the C entry point it calls. Tensors may be passed as
torch tensors (their data_ptr() is used) or as raw integer addresses; streams as a
torch.cuda.Stream, a raw cudaStream_t integer, or None (the legacy default stream). A non-zero
status raises TasqError carrying tasq_last_error(). There is no fallback: if libtasq.so is
missing the import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtasq.so")

TASQ_OK = 0
TASQ_ERR_INVALID_ARG = 1
TASQ_ERR_CUDA = 2
TASQ_ERR_UNSUPPORTED_ARCH = 3
TASQ_ERR_WORKSPACE = 4
TASQ_ERR_TIMEOUT = 5

TASQ_OUT_F16 = 0
TASQ_OUT_BF16 = 1
TASQ_NVFP4 = 0            # schedule entry of an NVFP4 step
TASQ_NVFP4_RAW_ACC = 2    # tasq_debug_gemm_nvfp4: raw FP32 accumulators

TASQ_DEVICE_TIMEOUT_PRODUCER = 0x1
TASQ_DEVICE_TIMEOUT_MMA = 0x2
TASQ_DEVICE_TIMEOUT_MASK = 0x4
TASQ_DEVICE_TIMEOUT_EPILOGUE = 0x8
TASQ_DEVICE_TIMEOUT_DRAIN = 0x10
TASQ_DEVICE_TIMEOUT_PROLOGUE = 0x20
TASQ_DEVICE_BAD_BITS = 0x100

TASQ_MAX_KP = 16384
TASQ_DMPQ_MAX_LAYERS = 32
TASQ_GROUP_MAX = 4
TASQ_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


class TasqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"tasq status {status}: {message}")
        self.status = status
        self.message = message


class tasq_layer_desc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("w", ctypes.c_void_p), ("s_w", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python timestep_adaptive_bit_b200/build.py` "
            "(or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, u64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
    sigs = {
        "tasq_linear_create": [ctypes.POINTER(P), ctypes.POINTER(tasq_layer_desc), i32, i32, i32, i64, i32, P],
        "tasq_set_schedule": [P, P, P],
        "tasq_linear_forward": [P, P, i64, i64, i32, i32, P, i64, P],
        "tasq_linear_destroy": [P],
        "tasq_get_device_status": [P, ctypes.POINTER(ctypes.c_uint32), i32, P],
        "tasq_set_wait_limit": [P, u64],
        "tasq_layer_info": [P, i32, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "tasq_debug_quantize": [P, P, i64, i64, i32, P, P, P],
        "tasq_debug_gemm_s32": [P, P, i64, i32, i32, P, i64, P],
        "tasq_debug_gemm": [P, P, P, i64, i32, i32, P, i64, i32, P],
        "tasq_debug_stuck_wait": [P, P],
        "tasq_debug_set_gemm_mode": [P, i32],
        "tasq_gemm_choice": [i64, i32, i32, ctypes.POINTER(i32)],
        "tasq_nvfp4_gemm_choice": [i64, i32, i32, ctypes.POINTER(i32)],
        "tasq_nvfp4_scale_bytes": [i64, i32, ctypes.POINTER(i64)],
        "tasq_debug_quantize_nvfp4": [P, P, i64, i64, i32, P, P, P, P],
        "tasq_debug_nvfp4_weights": [P, i32, P, P, P],
        "tasq_debug_gemm_nvfp4": [P, P, P, P, i64, i32, P, i64, i32, P],
        "tasq_debug_set_mask_mode": [P, i32],
        "tasq_get_schedule": [P, P, P],
        "tasq_linear_forward_group": [P, P, i64, i64, P, i32, i32, P, P, P],
        "tasq_dmpq_update": [P, P, i64, P, i64, i64, i32, P, i32, i32, ctypes.c_double, i32, i32, P, P],
        "tasq_debug_set_prologue_mode": [P, i32],
        "tasq_trace_enable": [P, i32],
        "tasq_linear_forward_noalloc": [P, i64, i64, i32, P, P, i32, i32, i32, P, i64, i32, P, P],
        "tasq_noalloc_device_status": [ctypes.POINTER(ctypes.c_uint32), i32, P],
        "tasq_trace_read": [P, ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i32),
                            ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                            ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)],
    }
    for name, args in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.tasq_last_error.argtypes = []
    lib.tasq_last_error.restype = ctypes.c_char_p
    return lib


lib = _load()


def tasq_last_error() -> str:
    return lib.tasq_last_error().decode(errors="replace")


def _check(status: int) -> None:
    if status != TASQ_OK:
        raise TasqError(status, tasq_last_error())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return int(t.data_ptr())
    if isinstance(t, np.ndarray):
        return int(t.ctypes.data)
    raise TypeError(f"cannot take the address of {type(t)}")


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    if hasattr(s, "cuda_stream"):
        return int(s.cuda_stream)
    raise TypeError(f"not a stream: {type(s)}")


class Context:
    """Opaque tasq_ctx* handle (frees itself when garbage-collected if not destroyed)."""

    def __init__(self, handle: int, layers: Sequence[tuple], num_steps: int = 1):
        self.handle = handle
        self.layers = [(int(N), int(K)) for N, K, *_ in layers]
        self.num_steps = int(num_steps)

    @property
    def _as_parameter_(self):
        return ctypes.c_void_p(self.handle)

    def __del__(self):
        if getattr(self, "handle", None):
            try:
                lib.tasq_linear_destroy(ctypes.c_void_p(self.handle))
            except Exception:
                pass
            self.handle = None


def tasq_linear_create(layers: Iterable[tuple], num_steps: int, hadamard_n: int, max_tokens: int,
                       out_dtype: int = TASQ_OUT_F16, stream=None) -> Context:
    """layers: iterable of (N, K, w, s_w) with w [N, Kp] int8 and s_w [N] float32 (host numpy
    arrays or device tensors)."""
    layers = list(layers)
    arr = (tasq_layer_desc * len(layers))()
    keep = []
    for i, (N, K, w, s_w) in enumerate(layers):
        if isinstance(w, np.ndarray):
            w = np.ascontiguousarray(w, dtype=np.int8)
            keep.append(w)
        if isinstance(s_w, np.ndarray):
            s_w = np.ascontiguousarray(s_w, dtype=np.float32)
            keep.append(s_w)
        arr[i] = tasq_layer_desc(int(N), int(K), _ptr(w), _ptr(s_w))
    h = ctypes.c_void_p()
    _check(lib.tasq_linear_create(ctypes.byref(h), arr, len(layers), int(num_steps), int(hadamard_n),
                                  int(max_tokens), int(out_dtype), _stream(stream)))
    del keep
    return Context(h.value, layers, num_steps)


def tasq_set_schedule(ctx: Context, bits, stream=None) -> None:
    b = np.ascontiguousarray(bits, dtype=np.uint8)
    _check(lib.tasq_set_schedule(ctx, b.ctypes.data, _stream(stream)))


def tasq_linear_forward(ctx: Context, x, M: int, ldx: int, layer: int, step: int, y, ldy: int, stream=None) -> None:
    _check(lib.tasq_linear_forward(ctx, _ptr(x), int(M), int(ldx), int(layer), int(step), _ptr(y), int(ldy),
                                   _stream(stream)))


def tasq_linear_forward_group(ctx: Context, x, M: int, ldx: int, layers, step: int, ys, ldys, stream=None) -> None:
    idx = np.ascontiguousarray(np.asarray(list(layers), dtype=np.int32))
    ptrs = (ctypes.c_void_p * len(ys))(*[_ptr(y) for y in ys])
    lds = np.ascontiguousarray(np.asarray(list(ldys), dtype=np.int64))
    if not (idx.size == len(ys) == lds.size):
        raise ValueError("layers, ys and ldys must have the same length")
    _check(lib.tasq_linear_forward_group(ctx, _ptr(x), int(M), int(ldx), idx.ctypes.data, int(idx.size), int(step),
                                         ctypes.cast(ptrs, ctypes.c_void_p), lds.ctypes.data, _stream(stream)))


def tasq_get_schedule(ctx: Context, stream=None) -> np.ndarray:
    """The device schedule table as a host uint8 array [num_layers, num_steps]."""
    n = (len(ctx.layers), ctx.num_steps)
    out = np.empty(n, dtype=np.uint8)
    _check(lib.tasq_get_schedule(ctx, out.ctypes.data, _stream(stream)))
    return out


def tasq_dmpq_update(ctx: Context, block_in, ld_in: int, block_out, ld_out: int, M: int, D: int, layers, step: int,
                     tau: float, bits_unstable: int, bits_stable: int, gamma_out=None, stream=None) -> None:
    idx = np.ascontiguousarray(np.asarray(list(layers), dtype=np.int32))
    _check(lib.tasq_dmpq_update(ctx, _ptr(block_in), int(ld_in), _ptr(block_out), int(ld_out), int(M), int(D),
                                idx.ctypes.data, int(idx.size), int(step), float(tau), int(bits_unstable),
                                int(bits_stable), _ptr(gamma_out), _stream(stream)))


def tasq_linear_destroy(ctx: Context) -> None:
    if ctx.handle:
        h, ctx.handle = ctx.handle, None
        _check(lib.tasq_linear_destroy(ctypes.c_void_p(h)))


def tasq_get_device_status(ctx: Context, clear: bool = False, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(lib.tasq_get_device_status(ctx, ctypes.byref(v), 1 if clear else 0, _stream(stream)))
    return int(v.value)


def tasq_set_wait_limit(ctx: Context, limit_ns: int) -> None:
    _check(lib.tasq_set_wait_limit(ctx, int(limit_ns)))


def tasq_layer_info(ctx: Context, layer: int):
    N, K, Kp = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib.tasq_layer_info(ctx, int(layer), ctypes.byref(N), ctypes.byref(K), ctypes.byref(Kp)))
    return int(N.value), int(K.value), int(Kp.value)


def tasq_debug_quantize(ctx: Context, x, M: int, ldx: int, layer: int, xq, s_x, stream=None) -> None:
    _check(lib.tasq_debug_quantize(ctx, _ptr(x), int(M), int(ldx), int(layer), _ptr(xq), _ptr(s_x), _stream(stream)))


def tasq_nvfp4_scale_bytes(rows: int, Kp: int) -> int:
    """Bytes of the NVFP4 block scales of `rows` rows with Kp in-features (host-only)."""
    out = ctypes.c_int64(0)
    _check(lib.tasq_nvfp4_scale_bytes(int(rows), int(Kp), ctypes.byref(out)))
    return int(out.value)


def tasq_debug_quantize_nvfp4(ctx: Context, x, M: int, ldx: int, layer: int, codes, scales, s_x,
                              stream=None) -> None:
    _check(lib.tasq_debug_quantize_nvfp4(ctx, _ptr(x), int(M), int(ldx), int(layer), _ptr(codes), _ptr(scales),
                                         _ptr(s_x), _stream(stream)))


def tasq_debug_nvfp4_weights(ctx: Context, layer: int, codes, scales, stream=None) -> None:
    _check(lib.tasq_debug_nvfp4_weights(ctx, int(layer), _ptr(codes), _ptr(scales), _stream(stream)))


def tasq_debug_gemm_nvfp4(ctx: Context, codes, scales, s_x, M: int, layer: int, y, ldy: int, out_kind: int,
                          stream=None) -> None:
    _check(lib.tasq_debug_gemm_nvfp4(ctx, _ptr(codes), _ptr(scales), _ptr(s_x), int(M), int(layer), _ptr(y),
                                     int(ldy), int(out_kind), _stream(stream)))


def tasq_debug_gemm_s32(ctx: Context, xq, M: int, layer: int, step: int, acc, ld_acc: int, stream=None) -> None:
    _check(lib.tasq_debug_gemm_s32(ctx, _ptr(xq), int(M), int(layer), int(step), _ptr(acc), int(ld_acc),
                                   _stream(stream)))


def tasq_debug_gemm(ctx: Context, xq, s_x, M: int, layer: int, step: int, y, ldy: int, out_dtype: int,
                    stream=None) -> None:
    _check(lib.tasq_debug_gemm(ctx, _ptr(xq), _ptr(s_x), int(M), int(layer), int(step), _ptr(y), int(ldy),
                               int(out_dtype), _stream(stream)))


def tasq_debug_set_gemm_mode(ctx: Context, mode: int) -> None:
    _check(lib.tasq_debug_set_gemm_mode(ctx, int(mode)))


def tasq_gemm_choice(M: int, N: int, num_sms: int) -> bool:
    """True when the automatic choice runs this GEMM on CTA pairs; host-only, needs no device."""
    pair = ctypes.c_int32(0)
    _check(lib.tasq_gemm_choice(int(M), int(N), int(num_sms), ctypes.byref(pair)))
    return bool(pair.value)


def tasq_nvfp4_gemm_choice(M: int, N: int, num_sms: int) -> bool:
    """True when the automatic choice runs this NVFP4 GEMM on CTA pairs; host-only."""
    pair = ctypes.c_int32(0)
    _check(lib.tasq_nvfp4_gemm_choice(int(M), int(N), int(num_sms), ctypes.byref(pair)))
    return bool(pair.value)


def tasq_debug_set_prologue_mode(ctx: Context, mode: int) -> None:
    _check(lib.tasq_debug_set_prologue_mode(ctx, int(mode)))


def tasq_debug_set_mask_mode(ctx: Context, mode: int) -> None:
    _check(lib.tasq_debug_set_mask_mode(ctx, int(mode)))


def tasq_debug_stuck_wait(ctx: Context, stream=None) -> None:
    _check(lib.tasq_debug_stuck_wait(ctx, _stream(stream)))


def tasq_trace_enable(ctx: Context, capacity: int) -> None:
    _check(lib.tasq_trace_enable(ctx, int(capacity)))


def tasq_trace_read(ctx: Context) -> dict:
    pl, gl = ctypes.c_int32(), ctypes.c_int32()
    pm, gm, ops, pb, wb = (ctypes.c_double() for _ in range(5))
    _check(lib.tasq_trace_read(ctx, ctypes.byref(pl), ctypes.byref(pm), ctypes.byref(gl), ctypes.byref(gm),
                               ctypes.byref(ops), ctypes.byref(pb), ctypes.byref(wb)))
    return {"prologue_launches": pl.value, "prologue_ms": pm.value, "gemm_launches": gl.value,
            "gemm_ms": gm.value, "gemm_ops": ops.value, "prologue_bytes": pb.value, "weight_pass_bytes": wb.value}


def tasq_linear_forward_noalloc(x, M: int, ldx: int, K: int, w, s_w, N: int, bits: int, hadamard_n: int, y,
                                ldy: int, out_dtype: int = TASQ_OUT_F16, device_status=None, stream=None) -> None:
    """Allocation-free forward: no context, the caller's weights are used in place and the
    activation workspace is a fixed device array inside the library (see include/tasq.h)."""
    _check(lib.tasq_linear_forward_noalloc(_ptr(x), int(M), int(ldx), int(K), _ptr(w), _ptr(s_w), int(N), int(bits),
                                           int(hadamard_n), _ptr(y), int(ldy), int(out_dtype), _ptr(device_status),
                                           _stream(stream)))


def tasq_noalloc_device_status(clear: bool = False, stream=None) -> int:
    """Status word of the allocation-free calls made without a device status pointer."""
    v = ctypes.c_uint32()
    _check(lib.tasq_noalloc_device_status(ctypes.byref(v), 1 if clear else 0, _stream(stream)))
    return int(v.value)
