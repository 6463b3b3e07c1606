"""Plain CPU oracle of the timestep-adaptive masked INT8 linear.

TEST INFRASTRUCTURE ONLY. This module is imported by tests/, by __graft_entry__.smoke() and by
bench.py's cpu_baseline / reference leg, and by nothing else. The product path (the CUDA
library and its Python binding) never imports it and shares no code with it.

It follows the pages step by step, slowly and in the open:

  1. Block Hadamard on the activations, z = X H with H block-diagonal of standard Hadamard
     matrices H_n (HQ-DM technical summary, section 2.1 "Mecanismo"; 6Bit-Diffusion section 2.A,
     "Suavizacao de Outliers" / Block Hadamard Transform). H_n is read as the Sylvester matrix,
     H_n[i, j] = (-1)^popcount(i & j), blocks are contiguous runs of n input channels, and rows
     are zero-padded to Kp = ceil(K / n) * n.
  2. The normalisation 2^(-k/2) = 1/sqrt(n) of H_n is kept out of the integer path and folded
     into the floating-point scale (HQ-DM section 2.1, "Eficiencia de Hardware").
  3. Symmetric per-token INT8 quantization of z (HQ-DM section 2.2, "Quantizacao Simetrica"),
     with a dynamic absmax scale per token and round-half-to-even codes in [-127, 127].
  4. The temporal-spatial LSB mask on the one shared 8-bit weight buffer, applied per (layer,
     step): Q^(t,l) = Q_n - (1 - M_t,l) * LSB, realised as dropping the k = 8 - bits lowest
     two's-complement bit planes (TASQ technical summary, section 2, "Representacao de Peso
     Compartilhada e Mascaramento de LSB" and its equation; the TASQ abstract on newx.sg).
  5. Integer GEMM, then FP dequantization by the per-token and per-channel scales (HQ-DM
     section 2.1, "Eficiencia de Hardware": the core computation is integer matrix products).

Precision: where floating point decides an integer (the INT8 activation codes), this oracle
takes the decision in FP32, the precision the method is specified in for the Hadamard, using
the textbook radix-2 fast Walsh-Hadamard butterfly in natural order. The exact FP64 transform is
kept beside it to pin it (for FP16 inputs the FP64 transform is exact). Everything after the
codes is exact integer arithmetic, then FP64 dequantization.
"""
from __future__ import annotations

import math
from typing import Dict

import numpy as np

INT8_QMAX = 127


# --------------------------------------------------------------------------------------------
# step 1: block Hadamard
# --------------------------------------------------------------------------------------------
def sylvester_hadamard(n: int) -> np.ndarray:
    """Standard (Sylvester, natural-order) Hadamard matrix H_n as int64, entries +-1.

    H_n[i, j] = (-1)^popcount(i & j). HQ-DM section 2.1 builds the block-diagonal H from standard
    Hadamard matrices H_k; this is the standard construction for n a power of two."""
    if n < 1 or n & (n - 1):
        raise ValueError("n must be a power of two")
    i = np.arange(n, dtype=np.int64)[:, None]
    j = np.arange(n, dtype=np.int64)[None, :]
    bits = i & j
    parity = np.zeros_like(bits)
    while np.any(bits):
        parity ^= bits & 1
        bits >>= 1
    return np.where(parity == 0, 1, -1).astype(np.int64)


def padded_k(K: int, n: int) -> int:
    return -(-K // n) * n


def pad_rows(x: np.ndarray, n: int) -> np.ndarray:
    """Zero-pad each row of x [M, K] to Kp = ceil(K / n) * n columns (float64 copy)."""
    M, K = x.shape
    out = np.zeros((M, padded_k(K, n)), dtype=np.float64)
    out[:, :K] = x.astype(np.float64)
    return out


def block_hadamard_exact(x: np.ndarray, n: int) -> np.ndarray:
    """z = x_pad . blockdiag(H_n, ..., H_n) in FP64.

    Exact for FP16 inputs: every FP16 value is a multiple of 2^-24 below 2^16 in magnitude, so
    every partial sum of at most n <= 2^7 such terms is a multiple of 2^-24 below 2^23 and needs
    at most 47 significant bits < 53. The summation order therefore does not matter."""
    xp = pad_rows(x, n)
    M, Kp = xp.shape
    H = sylvester_hadamard(n).astype(np.float64)
    z = xp.reshape(M, Kp // n, n) @ H
    return z.reshape(M, Kp)


def block_hadamard_fp32(x: np.ndarray, n: int) -> np.ndarray:
    """z = x_pad . blockdiag(H_n) computed in FP32 by the textbook fast Walsh-Hadamard transform.

    For h = 1, 2, 4, ..., n/2, every pair of entries (j, j + h) of a block with (j & h) == 0 is
    replaced by (a + b, a - b). After log2(n) stages this is x . H_n with H_n in Sylvester order.
    Each addition is one IEEE FP32 round-to-nearest operation."""
    xp = pad_rows(x, n).astype(np.float32)
    M, Kp = xp.shape
    z = xp.reshape(M, Kp // n, n).copy()
    h = 1
    while h < n:
        zz = z.reshape(M, Kp // n, n // (2 * h), 2, h)
        a = zz[:, :, :, 0, :].copy()
        b = zz[:, :, :, 1, :].copy()
        zz[:, :, :, 0, :] = a + b
        zz[:, :, :, 1, :] = a - b
        z = zz.reshape(M, Kp // n, n)
        h *= 2
    return z.reshape(M, Kp)


# --------------------------------------------------------------------------------------------
# steps 2-3: per-token symmetric INT8 quantization with the 1/sqrt(n) extracted into the scale
# --------------------------------------------------------------------------------------------
def quantize_per_token(z32: np.ndarray, n: int):
    """Codes q [M, Kp] int8 and scales s_x [M] float64 from the FP32 transform z32 [M, Kp].

    a     = max_k |z[m, k]|                      (exact in FP32)
    q     = clamp(RNE(z * fp32(127 / a)), -127, 127), all zero when a == 0
    s_x   = a / (127 * sqrt(n))                 (the extracted 2^(-k/2) of HQ-DM section 2.1)
    so that z / sqrt(n) ~= s_x * q. The reciprocal 127 / a is one FP32 division and the product
    with z one FP32 multiply, both round-to-nearest-even; np.rint rounds halves to even."""
    z32 = np.asarray(z32, dtype=np.float32)
    a = np.max(np.abs(z32), axis=1)
    q = np.zeros(z32.shape, dtype=np.int8)
    live = a > 0
    inv = np.zeros_like(a)
    inv[live] = np.float32(INT8_QMAX) / a[live]
    t = z32 * inv[:, None]                    # float32 * float32 -> float32
    codes = np.clip(np.rint(t), -INT8_QMAX, INT8_QMAX)
    q[live] = codes[live].astype(np.int8)
    s_x = a.astype(np.float64) / (INT8_QMAX * math.sqrt(n))
    return q, s_x, a


def prologue(x: np.ndarray, n: int):
    """Block Hadamard + per-token INT8 quantization of FP16 activations x [M, K]."""
    z32 = block_hadamard_fp32(x, n)
    q, s_x, a = quantize_per_token(z32, n)
    return q, s_x, z32


# --------------------------------------------------------------------------------------------
# step 4: temporal-spatial LSB mask
# --------------------------------------------------------------------------------------------
def lsb_mask(w: np.ndarray, bits: int) -> np.ndarray:
    """W_k = W with its k = 8 - bits least-significant two's-complement bit planes cleared.

    TASQ section 2: the operative weight at (stage t, layer l) is the shared 8-bit weight with
    LSBs truncated (bit-plane truncation or right shift). Clearing the planes equals
    (W >> k) << k with an arithmetic shift, i.e. 2^k * floor(W / 2^k). bits = 8 is the identity."""
    if not 1 <= int(bits) <= 8:
        raise ValueError("bits must be in [1, 8]")
    k = 8 - int(bits)
    keep = np.uint8((0xFF << k) & 0xFF)
    return (np.asarray(w, dtype=np.int8).view(np.uint8) & keep).view(np.int8)


# --------------------------------------------------------------------------------------------
# step 5: integer GEMM and dequantization
# --------------------------------------------------------------------------------------------
def int_gemm(q: np.ndarray, wk: np.ndarray) -> np.ndarray:
    """acc[m, j] = sum_c q[m, c] * wk[j, c], exact, as int64.

    Computed as an FP64 matrix product of integer-valued arrays: every partial sum is an integer
    of magnitude at most 127 * 128 * Kp < 2^31, hence exactly representable, so the result is
    exact in any summation order."""
    Kp = q.shape[1]
    if wk.shape[1] != Kp:
        raise ValueError("inner dimensions differ")
    if 127 * 128 * Kp >= 2 ** 31:
        raise ValueError("Kp too large for an int32 accumulator")
    acc = q.astype(np.float64) @ wk.astype(np.float64).T
    return np.rint(acc).astype(np.int64)


def dequant(acc: np.ndarray, s_x: np.ndarray, s_w: np.ndarray) -> np.ndarray:
    """y[m, j] = acc[m, j] * s_x[m] * s_w[j] in FP64."""
    return acc.astype(np.float64) * np.asarray(s_x, np.float64)[:, None] * np.asarray(s_w, np.float64)[None, :]


def masked_linear(x: np.ndarray, w: np.ndarray, s_w: np.ndarray, bits: int, n: int) -> Dict[str, np.ndarray]:
    """The whole path for one (layer, step): FP16 x [M, K], INT8 w [N, Kp], FP32 s_w [N]."""
    q, s_x, z32 = prologue(x, n)
    wk = lsb_mask(w, bits)
    acc = int_gemm(q, wk)
    y = dequant(acc, s_x, s_w)
    return {"z32": z32, "q": q, "s_x": s_x, "wk": wk, "acc": acc, "y": y}


# --------------------------------------------------------------------------------------------
# BitOPs model (TASQ section 2, "Motor de Precisao Temporal": bit-serial cycles scale with the
# product of the weight and activation bit widths)
# --------------------------------------------------------------------------------------------
def bitops(M: int, N: int, K: int, w_bits: int, a_bits: int = 8) -> int:
    return int(M) * int(N) * int(K) * int(w_bits) * int(a_bits)


# --------------------------------------------------------------------------------------------
# next row: DMPQ-style precision predictor (6Bit-Diffusion section 2.A, "Quantizacao de
# Precisao Mista Dinamica (DMPQ)")
# --------------------------------------------------------------------------------------------
# The block's transformation magnitude at the previous step is the relative L1 distance between
# its input and output, Gamma_(t-1) = ||out - in||_1 / ||in||_1; a light predictor keeps the
# unstable layers (large Gamma) at 8 bits and compresses the stable ones. Readings:
#   * the predictor is a threshold tau on Gamma: bits = hi if Gamma > tau else lo;
#   * both norms are taken over every element of the block's FP16 input and output (same shape);
#   * ||in||_1 = 0 carries no information, so the layer stays unstable (hi);
#   * the two L1 sums are exact (every FP16 value is an integer multiple of 2^-24), and Gamma is
#     their quotient in IEEE double: each sum rounded once to double, then one division.

def fp16_units(x: np.ndarray) -> np.ndarray:
    """FP16 values as exact integers in units of 2^-24 (the smallest FP16 subnormal), int64."""
    x = np.asarray(x)
    assert x.dtype == np.float16, "DMPQ inputs are FP16"
    assert np.all(np.isfinite(x)), "non-finite inputs are outside the method"
    return (x.astype(np.float64) * 2.0 ** 24).astype(np.int64)   # |x| < 2^16: exact


def _exact_sum(a: np.ndarray) -> int:
    """Sum of non-negative int64 values as a Python integer, in int64 chunks that cannot overflow
    (each term < 2^41, so 2^20 terms stay below 2^61)."""
    flat = a.reshape(-1)
    total = 0
    for i in range(0, flat.size, 1 << 20):
        total += int(flat[i:i + (1 << 20)].sum(dtype=np.int64))
    return total


def dmpq_l1_sums(x_in: np.ndarray, x_out: np.ndarray):
    """(||out - in||_1, ||in||_1) exactly, in units of 2^-24, as Python integers."""
    assert x_in.shape == x_out.shape
    u_in = fp16_units(x_in)
    u_out = fp16_units(x_out)
    return _exact_sum(np.abs(u_out - u_in)), _exact_sum(np.abs(u_in))


def dmpq_gamma(x_in: np.ndarray, x_out: np.ndarray) -> float:
    """Gamma = ||out - in||_1 / ||in||_1 in IEEE double (each exact sum rounded once to double,
    one division); +inf when ||in||_1 = 0 and the output differs, 0 when both are 0."""
    num, den = dmpq_l1_sums(x_in, x_out)
    if den == 0:
        return math.inf if num > 0 else 0.0
    return float(num) / float(den)


def dmpq_bits(gamma: float, tau: float, bits_unstable: int, bits_stable: int, den_zero: bool = False) -> int:
    """The predictor's decision: unstable (Gamma > tau, or no information) keeps bits_unstable."""
    if den_zero or gamma > tau:
        return int(bits_unstable)
    return int(bits_stable)
