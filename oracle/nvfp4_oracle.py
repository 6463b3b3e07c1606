"""Plain CPU oracle of the NVFP4 branch for stable layers.

TEST INFRASTRUCTURE ONLY, like tasq_oracle: imported by tests/, __graft_entry__.smoke() and
bench.py's CPU legs, never by the product path, and sharing no code with the CUDA library.

6Bit-Diffusion (technical summary, section 2.A, "Quantizacao de Precisao Mista Dinamica
(DMPQ)") keeps the unstable layers of a step in INT8 and compresses the stable ones to NVFP4,
Blackwell's native 4-bit format, after the same block Hadamard transform of the activations.
The pages name the format and nothing more; what NVFP4 is comes from NVIDIA's public definition:

  * element: E2M1, one sign bit, two exponent bits (bias 1), one mantissa bit; magnitudes
    0, 0.5, 1, 1.5, 2, 3, 4, 6;
  * block scale: one unsigned E4M3 number (four exponent bits, bias 7, three mantissa bits,
    largest finite 448, subnormals down to 2^-9) per 16 consecutive elements along K;
  * a second-level FP32 scale. NVIDIA's recipe has one per tensor; here it is one per token for
    the activations and one per output channel for the weights, the same granularity as the
    INT8 path's s_x and s_w, so that the dequantizing epilogue is unchanged.

Readings taken where the pages are silent (all decisions that floating point takes are taken in
FP32, as in the INT8 path):

  activations (after the FP32 block Hadamard z of tasq_oracle.block_hadamard_fp32):
    a     = max |z| over the padded row
    g     = fp32(2688 / a)            2688 = 6 * 448, so every block scale below fits E4M3
    u     = fp32(z * g)
    per block of 16: b = max |u|, sb = E4M3_RNE(fp32(b / 6)) (saturating at 448),
                     r = fp32(1 / sb), e = E2M1_RNE(fp32(u * r)) (saturating at +-6);
                     a block whose scale is 0 gets all-zero codes
    s_x   = a / (2688 * sqrt(n))      so that z / sqrt(n) ~= s_x * sb * e
  weights: the same per 16-block steps on the shared INT8 buffer itself (no LSB mask: the
    NVFP4 step replaces the truncation), W ~= sb * e in INT8 units; s_w is unchanged.
  GEMM: acc[m, j] = sum over blocks of sa * sw * sum_k ea * ew, computed here exactly (every
    value is a multiple of 2^-10, so the sum is an exact integer number of 2^-20 units);
    the tensor core accumulates in FP32.
  output: y = acc * s_x[m] * s_w[j].

Codes are packed two per byte along K, the lower-indexed element in the low nibble (E2M1 code =
sign << 3 | exponent << 1 | mantissa). Block scales are E4M3 bytes with the sign bit clear.
"""
from __future__ import annotations

import math

import numpy as np

from .tasq_oracle import block_hadamard_fp32

NVFP4_BLOCK = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0
ACT_RANGE = E2M1_MAX * E4M3_MAX          # 2688: the token's absmax maps to the top of both ranges

# E2M1 magnitudes by 3-bit code (exponent << 1 | mantissa)
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    """Value of 4-bit E2M1 codes (sign in bit 3)."""
    c = np.asarray(code).astype(np.int64) & 0xF
    mag = E2M1_VALUES[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_encode(t: np.ndarray) -> np.ndarray:
    """Round FP values to the nearest E2M1 value, ties to the even mantissa bit, magnitudes above
    6 saturating to 6, the sign kept (so a negative value that rounds to zero gives -0, code 8);
    returns 4-bit codes (uint8). Written as a search over the eight magnitudes, with the tie
    rule applied where two are equally near."""
    t = np.asarray(t, dtype=np.float64)
    mag = np.minimum(np.abs(t), E2M1_MAX)
    d = np.abs(mag[..., None] - E2M1_VALUES)              # distance to every magnitude
    best = np.argmin(d, axis=-1)                          # the lower code wins a tie here ...
    dmin = np.take_along_axis(d, best[..., None], -1)[..., 0]
    nxt = np.minimum(best + 1, 7)
    dn = np.take_along_axis(d, nxt[..., None], -1)[..., 0]
    tie = (nxt != best) & (dn == dmin)
    # ... so on a tie take the neighbour when the lower one has an odd mantissa bit
    best = np.where(tie & ((best & 1) == 1), nxt, best)
    sign = np.signbit(t).astype(np.int64)       # IEEE: a negative value rounding to 0 gives -0
    return ((sign << 3) | best).astype(np.uint8)


def _e4m3_values() -> np.ndarray:
    """All 127 non-negative finite E4M3 values by 7-bit code (exponent << 3 | mantissa); code
    0x7F is NaN in E4M3 and is left out."""
    v = np.zeros(127)
    for c in range(127):
        e, m = c >> 3, c & 7
        v[c] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return v


E4M3_VALUES = _e4m3_values()


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """Value of unsigned E4M3 scale bytes (sign bit clear)."""
    c = np.asarray(code).astype(np.int64)
    if np.any(c >= 127):
        raise ValueError("not a finite non-negative E4M3 code")
    return E4M3_VALUES[c]


def e4m3_encode(s: np.ndarray) -> np.ndarray:
    """Round non-negative FP values to the nearest E4M3 value, ties to the even code, values
    above 448 saturating to 448; returns bytes."""
    s = np.asarray(s, dtype=np.float64)
    if np.any(s < 0) or not np.all(np.isfinite(s)):
        raise ValueError("scales must be finite and non-negative")
    s = np.minimum(s, E4M3_MAX)
    d = np.abs(s[..., None] - E4M3_VALUES)
    best = np.argmin(d, axis=-1)
    dmin = np.take_along_axis(d, best[..., None], -1)[..., 0]
    nxt = np.minimum(best + 1, 126)
    dn = np.take_along_axis(d, nxt[..., None], -1)[..., 0]
    tie = (nxt != best) & (dn == dmin)
    best = np.where(tie & ((best & 1) == 1), nxt, best)
    return best.astype(np.uint8)


def _quantize_blocks(u32: np.ndarray):
    """E2M1 codes and E4M3 block scales of FP32 values u32 [R, C] (C a multiple of 16), each
    block of 16 along a row scaled by its own E4M3 scale, following the steps in the header."""
    u32 = np.asarray(u32, dtype=np.float32)
    R, C = u32.shape
    if C % NVFP4_BLOCK:
        raise ValueError("row length must be a multiple of 16")
    blk = u32.reshape(R, C // NVFP4_BLOCK, NVFP4_BLOCK)
    b = np.max(np.abs(blk), axis=2)                                   # exact
    sb_code = e4m3_encode((b / np.float32(E2M1_MAX)).astype(np.float32).astype(np.float64))
    sb = e4m3_decode(sb_code).astype(np.float32)
    live = sb > 0
    r = np.zeros_like(sb)
    r[live] = np.float32(1.0) / sb[live]                              # one FP32 division
    t = blk * r[:, :, None]                                           # FP32 products
    codes = e2m1_encode(t.astype(np.float64))
    codes[~live] = 0
    return codes.reshape(R, C), sb_code


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[R, C] 4-bit codes -> [R, C/2] bytes, element 2i in the low nibble of byte i."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def quantize_activations(z32: np.ndarray, n: int):
    """NVFP4 codes [M, Kp] (unpacked 4-bit), block scales [M, Kp/16] (E4M3 bytes) and s_x [M]
    (float64) of the FP32 block-Hadamard output z32 [M, Kp]."""
    z32 = np.asarray(z32, dtype=np.float32)
    a = np.max(np.abs(z32), axis=1)
    g = np.zeros_like(a)
    live = a > 0
    g[live] = np.float32(ACT_RANGE) / a[live]                        # one FP32 division per token
    u = z32 * g[:, None]                                              # FP32 products
    codes, sb = _quantize_blocks(u)
    s_x = a.astype(np.float64) / (ACT_RANGE * math.sqrt(n))
    return codes, sb, s_x


def nvfp4_prologue(x: np.ndarray, n: int):
    """Block Hadamard (FP32 FWHT) + NVFP4 quantization of FP16 activations x [M, K]."""
    z32 = block_hadamard_fp32(x, n)
    codes, sb, s_x = quantize_activations(z32, n)
    return codes, sb, s_x, z32


def quantize_weights(w: np.ndarray):
    """NVFP4 codes [N, Kp] and block scales [N, Kp/16] of the shared INT8 weights w [N, Kp]."""
    return _quantize_blocks(np.asarray(w, dtype=np.int8).astype(np.float32))


def nvfp4_gemm(ca: np.ndarray, sa: np.ndarray, cw: np.ndarray, sw: np.ndarray) -> np.ndarray:
    """acc[m, j] = sum_b sa[m, b] sw[j, b] sum_{k in b} ea[m, k] ew[j, k], exactly, as float64
    (exact as long as it is below 2^53 units of 2^-20, which every case here is).

    E2M1 values are multiples of 1/2 and E4M3 values multiples of 2^-9, so 2e and 512 sb are
    integers. Each block's integer dot product of the doubled codes is exact in an FP64 matrix
    product (at most 16 * 12 * 12); the scaled block terms are summed in int64."""
    ea2 = np.rint(2.0 * e2m1_decode(ca)).astype(np.float64)           # [M, Kp], integers
    ew2 = np.rint(2.0 * e2m1_decode(cw)).astype(np.float64)           # [N, Kp]
    sa512 = np.rint(512.0 * e4m3_decode(sa)).astype(np.int64)          # [M, Kp/16]
    sw512 = np.rint(512.0 * e4m3_decode(sw)).astype(np.int64)          # [N, Kp/16]
    M, Kp = ea2.shape
    N = ew2.shape[0]
    if ew2.shape[1] != Kp:
        raise ValueError("inner dimensions differ")
    acc = np.zeros((M, N), dtype=np.int64)
    for blk in range(Kp // NVFP4_BLOCK):
        k = slice(blk * NVFP4_BLOCK, (blk + 1) * NVFP4_BLOCK)
        dot = np.rint(ea2[:, k] @ ew2[:, k].T).astype(np.int64)
        acc += dot * sa512[:, blk][:, None] * sw512[:, blk][None, :]
    return acc.astype(np.float64) * 2.0 ** -20


def nvfp4_abs_terms(ca, sa, cw, sw) -> np.ndarray:
    """sum over k of |term_k| for each output: the scale of the FP32 accumulation error bound."""
    ea = np.abs(e2m1_decode(ca))
    ew = np.abs(e2m1_decode(cw))
    sae = np.repeat(e4m3_decode(sa), NVFP4_BLOCK, axis=1)
    swe = np.repeat(e4m3_decode(sw), NVFP4_BLOCK, axis=1)
    return (ea * sae) @ (ew * swe).T


def nvfp4_linear(x: np.ndarray, w: np.ndarray, s_w: np.ndarray, n: int):
    """The NVFP4 step of one layer: FP16 x [M, K], shared INT8 w [N, Kp], FP32 s_w [N]."""
    ca, sa, s_x, z32 = nvfp4_prologue(x, n)
    cw, sw = quantize_weights(w)
    acc = nvfp4_gemm(ca, sa, cw, sw)
    y = acc * np.asarray(s_x, np.float64)[:, None] * np.asarray(s_w, np.float64)[None, :]
    return {"z32": z32, "ca": ca, "sa": sa, "s_x": s_x, "cw": cw, "sw": sw, "acc": acc, "y": y}
