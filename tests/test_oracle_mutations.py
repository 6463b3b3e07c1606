"""Planted mistakes in copies of the oracle's steps must each fail a pin.

Every mutation below is a plausible slip (a dropped term, a wrong sign or index, a transposed
or misordered operand, the wrong rounding); the corresponding pin must reject it. The mistakes
are planted in local CPU variants only."""
import math

import numpy as np
import pytest

import oracle
import pins


def _fails(check, *args):
    with pytest.raises(AssertionError):
        check(*args)


# ---------------------------------------------------------------- Hadamard matrix
def _h_flipped(n):
    H = oracle.sylvester_hadamard(n).copy()
    if n > 1:
        H[n - 1, n - 1] *= -1
    return H


def _h_sequency(n):
    # rows sorted by their number of sign changes (Walsh / sequency order)
    H = oracle.sylvester_hadamard(n)
    changes = [int(np.sum(H[r, 1:] != H[r, :-1])) for r in range(n)]
    return H[np.argsort(changes, kind="stable")]


def test_mutation_hadamard_sign():
    _fails(pins.check_hadamard_matrix, _h_flipped)


def test_mutation_hadamard_order():
    _fails(pins.check_hadamard_matrix, _h_sequency)


# ---------------------------------------------------------------- block transform
def _bh_normalised(x, n):
    return oracle.block_hadamard_exact(x, n) / math.sqrt(n)


def _bh_truncating(x, n):
    K = x.shape[1] // n * n
    return oracle.block_hadamard_exact(x[:, :K], n)


def _bh_interleaved(x, n):
    # blocks formed from strided channels instead of contiguous runs
    xp = oracle.pad_rows(x, n)
    M, Kp = xp.shape
    nb = Kp // n
    perm = np.arange(Kp).reshape(n, nb).T.reshape(-1)
    z = oracle.block_hadamard_exact(xp[:, perm], n)
    out = np.empty_like(z)
    out[:, perm] = z
    return out


def test_mutation_block_normalised():
    _fails(pins.check_block_hadamard_exact, _bh_normalised)


def test_mutation_block_truncating():
    _fails(pins.check_block_hadamard_exact, _bh_truncating)


def test_mutation_block_interleaved():
    _fails(pins.check_block_hadamard_exact, _bh_interleaved)


def _fwht32_swapped(x, n):
    xp = oracle.pad_rows(x, n).astype(np.float32)
    M, Kp = xp.shape
    z = xp.reshape(M, Kp // n, n).copy()
    h = 1
    while h < n:
        zz = z.reshape(M, Kp // n, n // (2 * h), 2, h)
        a = zz[:, :, :, 0, :].copy()
        b = zz[:, :, :, 1, :].copy()
        zz[:, :, :, 0, :] = a + b
        zz[:, :, :, 1, :] = b - a          # wrong sign
        z = zz.reshape(M, Kp // n, n)
        h *= 2
    return z.reshape(M, Kp)


def _fwht32_missing_stage(x, n):
    xp = oracle.pad_rows(x, n).astype(np.float32)
    M, Kp = xp.shape
    z = xp.reshape(M, Kp // n, n).copy()
    h = 2                                   # skips the h = 1 stage
    while h < n:
        zz = z.reshape(M, Kp // n, n // (2 * h), 2, h)
        a = zz[:, :, :, 0, :].copy()
        b = zz[:, :, :, 1, :].copy()
        zz[:, :, :, 0, :] = a + b
        zz[:, :, :, 1, :] = a - b
        z = zz.reshape(M, Kp // n, n)
        h *= 2
    return z.reshape(M, Kp)


def test_mutation_fwht32_sign():
    _fails(pins.check_block_hadamard_fp32, _fwht32_swapped, oracle.block_hadamard_exact)


def test_mutation_fwht32_stage():
    _fails(pins.check_block_hadamard_fp32, _fwht32_missing_stage, oracle.block_hadamard_exact)


# ---------------------------------------------------------------- quantizer
def _q_with(rounder=np.rint, qmax_div=127, sqrt_in_scale=True, clamp=127):
    def quantize(z32, n):
        z32 = np.asarray(z32, dtype=np.float32)
        a = np.max(np.abs(z32), axis=1)
        q = np.zeros(z32.shape, dtype=np.int16)
        live = a > 0
        inv = np.zeros_like(a)
        inv[live] = np.float32(qmax_div) / a[live]
        codes = np.clip(rounder(z32 * inv[:, None]), -clamp, clamp)
        q[live] = codes[live]
        s_x = a.astype(np.float64) / (127 * (math.sqrt(n) if sqrt_in_scale else 1.0))
        return q.astype(np.int8) if clamp <= 127 else q, s_x, a
    return quantize


def _q_asymmetric(z32, n):
    z32 = np.asarray(z32, dtype=np.float32)
    lo, hi = z32.min(1), z32.max(1)
    rngv = np.where(hi > lo, hi - lo, 1).astype(np.float32)
    q = np.clip(np.rint((z32 - lo[:, None]) * (254 / rngv)[:, None]) - 127, -127, 127).astype(np.int8)
    a = np.max(np.abs(z32), axis=1)
    return q, a.astype(np.float64) / (127 * math.sqrt(n)), a


def test_mutation_quant_floor():
    _fails(pins.check_quantizer, _q_with(rounder=np.floor))


def test_mutation_quant_half_away():
    _fails(pins.check_quantizer, _q_with(rounder=lambda t: np.sign(t) * np.floor(np.abs(t) + 0.5)))


def test_mutation_quant_scale_without_sqrt():
    _fails(pins.check_quantizer, _q_with(sqrt_in_scale=False))


def test_mutation_quant_128_levels():
    _fails(pins.check_quantizer, _q_with(qmax_div=128, clamp=128))


def test_mutation_quant_asymmetric():
    _fails(pins.check_quantizer, _q_asymmetric)


# ---------------------------------------------------------------- mask
def _mask_round(w, bits):
    k = 8 - bits
    v = np.asarray(w, dtype=np.int64)
    r = np.clip(np.rint(v / (1 << k)) * (1 << k), -128, 127)
    return r.astype(np.int8)


def _mask_off_by_one(w, bits):
    return oracle.lsb_mask(w, max(bits - 1, 1)) if bits < 8 else np.asarray(w, np.int8)


def _mask_logical_shift(w, bits):
    k = 8 - bits
    u = np.asarray(w, dtype=np.int8).view(np.uint8).astype(np.int64)
    v = ((u >> k) << k)
    return np.where(np.asarray(w) < 0, -v, v).clip(-128, 127).astype(np.int8)


def test_mutation_mask_round():
    _fails(pins.check_mask, _mask_round)


def test_mutation_mask_off_by_one():
    _fails(pins.check_mask, _mask_off_by_one)


def test_mutation_mask_sign_magnitude():
    _fails(pins.check_mask, _mask_logical_shift)


# ---------------------------------------------------------------- GEMM + dequant
def _gemm_drop_tail(q, w):
    K = q.shape[1]
    return oracle.int_gemm(q[:, : K - 32], w[:, : K - 32])


def _gemm_int16(q, w):
    return (q.astype(np.int16) @ w.astype(np.int16).T).astype(np.int64)


def _gemm_transposed_weight_rows(q, w):
    return oracle.int_gemm(q, w[::-1])


def test_mutation_gemm_tail():
    _fails(pins.check_gemm, _gemm_drop_tail)


def test_mutation_gemm_overflow():
    _fails(pins.check_gemm, _gemm_int16)


def test_mutation_gemm_row_order():
    _fails(pins.check_gemm, _gemm_transposed_weight_rows)


def test_mutation_dequant_missing_sw():
    _fails(pins.check_dequant, lambda acc, sx, sw: acc * np.asarray(sx)[:, None])


def test_mutation_dequant_axes_swapped():
    _fails(pins.check_dequant, lambda acc, sx, sw: acc * np.asarray(sx)[None, :] * np.asarray(sw)[:, None])


def test_mutation_end_to_end_missing_sqrt():
    def linear(x, w, s_w, bits, n):
        out = oracle.masked_linear(x, w, s_w, bits, n)
        out = dict(out)
        out["y"] = out["y"] * math.sqrt(n)
        out["s_x"] = out["s_x"] * math.sqrt(n)
        return out
    _fails(pins.check_end_to_end, linear, oracle.block_hadamard_exact, oracle.sylvester_hadamard)


def test_mutation_end_to_end_unmasked():
    def linear(x, w, s_w, bits, n):
        out = dict(oracle.masked_linear(x, w, s_w, bits, n))
        out["y"] = oracle.dequant(oracle.int_gemm(out["q"], w), out["s_x"], s_w)
        return out
    _fails(pins.check_end_to_end, linear, oracle.block_hadamard_exact, oracle.sylvester_hadamard)


# ---------------------------------------------------------------- DMPQ predictor
def _g_l2(x_in, x_out):
    a = x_in.astype(np.float64)
    b = x_out.astype(np.float64)
    d = np.linalg.norm(a)
    return float(np.linalg.norm(b - a) / d) if d > 0 else (math.inf if np.any(b != a) else 0.0)


def _g_relative_to_output(x_in, x_out):
    return oracle.dmpq_gamma(x_out, x_in)


def _g_no_abs(x_in, x_out):
    a = x_in.astype(np.float64)
    b = x_out.astype(np.float64)
    d = float(np.abs(a).sum())
    return float(abs((b - a).sum()) / d) if d > 0 else (math.inf if np.any(b != a) else 0.0)


def _g_fp16_sums(x_in, x_out):
    d = np.abs(x_in).sum(dtype=np.float16)
    n = np.abs((x_out - x_in).astype(np.float16)).sum(dtype=np.float16)
    return float(n) / float(d) if d > 0 else (math.inf if n > 0 else 0.0)


def _bits_ge(gamma, tau, hi, lo, den_zero=False):
    return hi if (den_zero or gamma >= tau) else lo


def _bits_zero_stable(gamma, tau, hi, lo, den_zero=False):
    return hi if gamma > tau else lo


@pytest.mark.parametrize("gamma_fn", [_g_l2, _g_relative_to_output, _g_no_abs, _g_fp16_sums])
def test_mutation_dmpq_gamma(gamma_fn):
    _fails(pins.check_dmpq, gamma_fn, oracle.dmpq_bits, oracle.dmpq_l1_sums)


@pytest.mark.parametrize("bits_fn", [_bits_ge, _bits_zero_stable])
def test_mutation_dmpq_decision(bits_fn):
    _fails(pins.check_dmpq, oracle.dmpq_gamma, bits_fn, oracle.dmpq_l1_sums)


# ---------------------------------------------------------------- NVFP4 branch
def _e2m1_ties_away(t):
    # ties away from zero instead of to the even mantissa
    t = np.asarray(t, dtype=np.float64)
    grid = oracle.E2M1_VALUES
    mag = np.minimum(np.abs(t), 6.0)
    best = np.array([int(np.flatnonzero(np.abs(grid - v) == np.abs(grid - v).min())[-1]) for v in mag.ravel()])
    best = best.reshape(mag.shape)
    return ((np.signbit(t).astype(np.int64) << 3) | best).astype(np.uint8)


def _e4m3_truncating(s):
    # rounds toward zero instead of to nearest
    s = np.minimum(np.asarray(s, dtype=np.float64), 448.0)
    v = oracle.E4M3_VALUES
    return np.array([int(np.flatnonzero(v <= x)[-1]) for x in s.ravel()], dtype=np.uint8).reshape(s.shape)


def _quant_range_4(z32, n):
    # block scale b / 4 instead of b / 6: the block absmax no longer maps to the top code
    import oracle.nvfp4_oracle as O
    z32 = np.asarray(z32, dtype=np.float32)
    a = np.abs(z32).max(1)
    g = np.where(a > 0, np.float32(2688) / np.where(a > 0, a, 1), 0).astype(np.float32)
    u = z32 * g[:, None]
    blk = u.reshape(u.shape[0], -1, 16)
    b = np.abs(blk).max(2)
    sbc = oracle.e4m3_encode((b / np.float32(4)).astype(np.float32).astype(np.float64))
    sb = oracle.e4m3_decode(sbc).astype(np.float32)
    r = np.where(sb > 0, np.float32(1) / np.where(sb > 0, sb, 1), 0).astype(np.float32)
    codes = oracle.e2m1_encode((blk * r[:, :, None]).astype(np.float64)).reshape(u.shape)
    return codes, sbc, a.astype(np.float64) / (O.ACT_RANGE * math.sqrt(n))


def _gemm_without_weight_scales(ca, sa, cw, sw):
    return oracle.nvfp4_gemm(ca, sa, cw, np.full_like(sw, 0x38))   # every weight scale 1.0


def test_mutation_e2m1_ties_away():
    _fails(pins.check_e2m1, _e2m1_ties_away, oracle.e2m1_decode)


def test_mutation_e4m3_truncation():
    _fails(pins.check_e4m3, _e4m3_truncating, oracle.e4m3_decode)


def test_mutation_nvfp4_scale_range():
    _fails(pins.check_nvfp4_quantizer, _quant_range_4)


def test_mutation_nvfp4_gemm_drops_weight_scales():
    _fails(pins.check_nvfp4_gemm, _gemm_without_weight_scales)
