"""Pins for the oracle: checks against what the pages and the mathematics fix.

Each check takes the oracle functions it exercises as arguments, so the mutation tests can
hand it a deliberately broken variant and confirm that the check catches the mistake.
Every check raises AssertionError on failure.
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


# ------------------------------------------------------------------------ Hadamard matrix
def check_hadamard_matrix(sylvester):
    # golden H_4 written out by hand
    H4 = np.array([[int(v) for v in r.split()] for r in _golden_rows("hadamard_n4.txt")])
    assert np.array_equal(sylvester(4), H4), "H_4 differs from the hand-written Sylvester matrix"
    # Sylvester recursion H_2n = [[H, H], [H, -H]] from H_1 = [1]
    H = np.array([[1]])
    for n in (2, 4, 8, 16, 32, 64, 128):
        H = np.block([[H, H], [H, -H]])
        assert np.array_equal(sylvester(n), H), f"H_{n} breaks the Sylvester recursion"
    for n in (1, 2, 4, 8, 16, 32, 64, 128):
        Hn = sylvester(n).astype(np.int64)
        assert np.array_equal(Hn @ Hn.T, n * np.eye(n, dtype=np.int64)), f"H_{n} H_{n}^T != n I"
        assert np.array_equal(Hn, Hn.T), f"H_{n} not symmetric"


# ------------------------------------------------------------------------ block transform
def check_block_hadamard_exact(block_h):
    # golden worked examples
    for row in _golden_rows("fwht_examples.txt"):
        n_s, x_s, z_s = [p.strip() for p in row.split("|")]
        n = int(n_s)
        x = np.array([[float(v) for v in x_s.split()]], dtype=np.float16)
        z = np.array([[float(v) for v in z_s.split()]])
        assert np.array_equal(block_h(x, n), z), f"worked example n={n} x={x_s} differs"
    rng = np.random.default_rng(5)
    for n in (4, 64, 128):
        K = 3 * n
        # basis vectors give the rows of H (pins the ordering)
        H = np.array([[(-1) ** bin(i & j).count("1") for j in range(n)] for i in range(n)], dtype=np.float64)
        for i in (0, 1, n // 2 + 1, n - 1):
            e = np.zeros((1, K), dtype=np.float16)
            e[0, n + i] = 1.0            # second block
            z = block_h(e, n)
            assert np.array_equal(z[0, n:2 * n], H[i]), f"e_{i} does not map to row {i} of H_{n}"
            assert not np.any(z[0, :n]) and not np.any(z[0, 2 * n:]), "blocks leak into each other"
        # applying the transform twice returns n * x (H H = n I)
        x = rng.standard_normal((5, K)).astype(np.float16)
        z = block_h(x, n)
        z2 = block_h(z, n)
        assert np.allclose(z2, n * x.astype(np.float64), rtol=0, atol=1e-9 * n), "H H != n I on data"
        # Parseval: sum z^2 = n sum x^2
        assert np.allclose((z ** 2).sum(1), n * (x.astype(np.float64) ** 2).sum(1), rtol=1e-12)
    # zero padding of a ragged K: K = 1.5 blocks behaves like an explicit zero tail
    n = 64
    x = rng.standard_normal((3, 96)).astype(np.float16)
    xp = np.zeros((3, 128), dtype=np.float16)
    xp[:, :96] = x
    assert np.array_equal(block_h(x, n), block_h(xp, n)), "ragged K is not zero-padded"
    assert block_h(x, n).shape == (3, 128)


def check_block_hadamard_fp32(block_h32, block_h_exact):
    rng = np.random.default_rng(7)
    for n in (64, 128):
        # small integers: every butterfly is exact in FP32, so FP32 == FP64 exactly
        xi = rng.integers(-50, 51, size=(7, 2 * n)).astype(np.float16)
        assert np.array_equal(block_h32(xi, n).astype(np.float64), block_h_exact(xi, n))
        # FP16 data with outliers: error within the FP32 butterfly bound log2(n) * 2^-24 * sum|x|
        x = rng.standard_normal((16, 3 * n)).astype(np.float32)
        x[:, 5] *= 50
        x = x.astype(np.float16)
        z32 = block_h32(x, n).astype(np.float64)
        z64 = block_h_exact(x, n)
        l1 = np.abs(x.astype(np.float64)).reshape(16, 3, n).sum(-1).repeat(n, axis=1)
        bound = math.log2(n) * 2.0 ** -24 * l1
        assert np.all(np.abs(z32 - z64) <= bound), "FP32 transform outside its rounding bound"
        assert block_h32(x, n).dtype == np.float32


# ------------------------------------------------------------------------ quantizer
def check_quantizer(quantize):
    for row in _golden_rows("quant_examples.txt"):
        z_s, q_s, s_s = [p.strip() for p in row.split("|")]
        z = np.array([[float(v) for v in z_s.split()]], dtype=np.float32)
        q, s_x, a = quantize(z, 64)
        assert np.array_equal(q[0].astype(np.int64), np.array([int(v) for v in q_s.split()])), f"codes for {z_s}"
        assert s_x[0] == float(s_s), f"scale for {z_s}"
        assert q.dtype == np.int8
    rng = np.random.default_rng(11)
    z = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 100, size=(64, 1))).astype(np.float32)
    z[3] = 0.0
    q, s_x, a = quantize(z, 64)
    qi = q.astype(np.int64)
    assert qi.min() >= -127 and qi.max() <= 127, "codes outside [-127, 127]"
    assert not np.any(qi[3]) and s_x[3] == 0.0, "zero row must give zero codes and scale"
    live = np.arange(64) != 3
    # the absmax entry maps to +-127; codes reconstruct z within half a step
    assert np.all(np.abs(qi[live]).max(1) == 127)
    step = (a[live].astype(np.float64) / 127.0)[:, None]
    err = np.abs(qi[live] * step - z[live].astype(np.float64))
    assert np.all(err <= 0.5 * step * (1 + 1e-5)), "codes further than half a step from z"
    # scale carries the 1/sqrt(n): s_x * q ~= z / sqrt(n)
    for n in (64, 128):
        q, s_x, a = quantize(z, n)
        assert np.allclose(s_x[live], a[live].astype(np.float64) / (127 * math.sqrt(n)), rtol=1e-15)
    # sign symmetry
    qn, _, _ = quantize(-z, 64)
    assert np.array_equal(qn.astype(np.int64), -qi), "quantizer is not symmetric"


# ------------------------------------------------------------------------ LSB mask
def check_mask(mask):
    for row in _golden_rows("mask_examples.txt"):
        w, bits, r = (int(v) for v in row.split())
        got = int(mask(np.array([w], dtype=np.int8), bits)[0])
        assert got == r, f"mask({w}, {bits}) = {got}, expected {r}"
    allw = np.arange(-128, 128, dtype=np.int64)
    w8 = allw.astype(np.int8)
    assert np.array_equal(mask(w8, 8).astype(np.int64), allw), "bits = 8 must be the identity"
    for bits in range(1, 9):
        k = 8 - bits
        r = mask(w8, bits).astype(np.int64)
        assert np.all(r % (1 << k) == 0), "result not divisible by 2^k"
        assert np.all(r <= allw) and np.all(allw - r < (1 << k)), "not a floor truncation"
        floor = np.array([(int(v) // (1 << k)) * (1 << k) for v in allw])
        assert np.array_equal(r, floor), "differs from 2^k floor(w / 2^k)"
        assert len(np.unique(r)) == 1 << bits, "wrong number of representable levels"


# ------------------------------------------------------------------------ GEMM + dequant
def check_gemm(gemm):
    rng = np.random.default_rng(13)
    for (M, N, K) in ((1, 1, 64), (3, 4, 64), (4, 2, 128), (2, 3, 192)):
        q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
        w = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
        acc = gemm(q, w)
        brute = [[sum(int(q[m, c]) * int(w[j, c]) for c in range(K)) for j in range(N)] for m in range(M)]
        assert np.array_equal(np.asarray(acc, dtype=np.int64), np.array(brute, dtype=np.int64)), "GEMM != brute force"
    # the largest magnitude an int32 accumulator may see at Kp = 12288
    K = 12288
    q = np.full((1, K), -127, dtype=np.int8)
    w = np.full((2, K), -128, dtype=np.int8)
    w[1] = 127
    acc = np.asarray(gemm(q, w), dtype=np.int64)
    assert acc[0, 0] == 127 * 128 * K and acc[0, 1] == -127 * 127 * K
    assert abs(acc[0, 0]) < 2 ** 31


def check_dequant(dq):
    acc = np.array([[1000, -3], [0, 2 ** 30]], dtype=np.int64)
    s_x = np.array([0.5, 0.25])
    s_w = np.array([0.004, 2.0])
    y = dq(acc, s_x, s_w)
    expect = np.array([[2.0, -3.0], [0.0, 2.0 ** 29]])
    assert np.allclose(y, expect, rtol=1e-15, atol=0), "dequant closed form"


def check_end_to_end(linear, block_h_exact, sylvester):
    """With the stored weights read in the rotated basis, y approximates (X H / sqrt(n)) (s_w W_k)^T:
    the only gap is the activation quantization error, a fraction of a code step."""
    rng = np.random.default_rng(17)
    n, M, K, N = 64, 32, 160, 24
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, 7] *= 50
    x = x.astype(np.float16)
    Kp = -(-K // n) * n
    w = rng.integers(-127, 128, size=(N, Kp)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    for bits in (8, 5, 3):
        out = linear(x, w, s_w, bits, n)
        z = block_h_exact(x, n)
        wk = np.asarray(out["wk"], dtype=np.float64)
        real = (z / math.sqrt(n)) @ (s_w.astype(np.float64)[:, None] * wk).T
        rel = np.linalg.norm(out["y"] - real) / np.linalg.norm(real)
        assert rel < 0.02, f"end-to-end relative error {rel} too large at bits={bits}"
        # and the per-element error is bounded by the code rounding: |z/sqrt(n) - s_x q| <= s_x/2
        row_l1 = np.abs(s_w.astype(np.float64)[:, None] * wk).sum(1)
        bound = 0.5 * np.asarray(out["s_x"])[:, None] * row_l1[None, :]
        assert np.all(np.abs(out["y"] - real) <= bound * (1 + 1e-6) + 1e-12), "element outside rounding bound"


# ------------------------------------------------------------------------ DMPQ predictor
def check_dmpq(gamma_fn, bits_fn, sums_fn):
    from fractions import Fraction

    for row in _golden_rows("dmpq_examples.txt"):
        a, b, c, g, want = (p.strip() for p in row.split("|"))
        x_in = np.array([float(v) for v in a.split()], dtype=np.float16)
        x_out = np.array([float(v) for v in b.split()], dtype=np.float16)
        tau, hi, lo = float(c.split()[0]), int(c.split()[1]), int(c.split()[2])
        gamma = gamma_fn(x_in, x_out)
        assert gamma == float(g), f"Gamma {gamma!r}, expected {g}"
        den_zero = sums_fn(x_in, x_out)[1] == 0
        assert bits_fn(gamma, tau, hi, lo, den_zero) == int(want), f"bits for row {row!r}"
    rng = np.random.default_rng(77)
    x = (rng.standard_normal((64, 48)) * 3).astype(np.float16)
    x[:, 5] *= 100
    x = x.astype(np.float16)
    # closed forms: identity, negation, zero output, exact doubling
    assert gamma_fn(x, x) == 0.0
    assert gamma_fn(x, -x) == 2.0
    assert gamma_fn(x, np.zeros_like(x)) == 1.0
    small = (x / 8).astype(np.float16)
    assert gamma_fn(small, (small * 2).astype(np.float16)) == 1.0
    # invariance under a common power-of-two scale (exact in FP16 away from the range ends)
    y = (x + rng.standard_normal(x.shape).astype(np.float16)).astype(np.float16)
    g0 = gamma_fn(small, (y / 8).astype(np.float16))
    assert gamma_fn((small * 4).astype(np.float16), (y / 2).astype(np.float16)) == g0
    # invariance under any permutation of the elements applied to both tensors
    perm = rng.permutation(x.size)
    assert gamma_fn(x.reshape(-1)[perm], y.reshape(-1)[perm]) == gamma_fn(x, y)
    # brute force with exact rationals on small tensors (sums below 2^53: one rounding)
    for trial in range(20):
        n = int(rng.integers(1, 40))
        xi = (rng.standard_normal(n) * 10 ** rng.uniform(-6, 3)).astype(np.float16)
        xo = (xi + rng.standard_normal(n).astype(np.float16) * np.float16(0.1)).astype(np.float16)
        num = sum(abs(Fraction(float(o)) - Fraction(float(i))) for i, o in zip(xi, xo))
        den = sum(abs(Fraction(float(i))) for i in xi)
        got_num, got_den = sums_fn(xi, xo)
        assert Fraction(got_num, 1 << 24) == num and Fraction(got_den, 1 << 24) == den, "inexact L1 sums"
        if den > 0:
            assert gamma_fn(xi, xo) == float(num / den), "Gamma is not the correctly rounded quotient"
    # a large tensor: the sums must not overflow (terms up to 2^41 units, 2^22 of them)
    big = np.full(1 << 22, 65504, dtype=np.float16)
    num, den = sums_fn(big, -big)
    assert den == 65504 * (1 << 24) * (1 << 22) and num == 2 * den


# ------------------------------------------------------------------------ NVFP4 branch
def check_e2m1(encode, decode):
    for row in _golden_rows("nvfp4_e2m1_examples.txt"):
        v, c = (p.strip() for p in row.split("|"))
        got = int(encode(np.array([float(v)]))[0])
        assert got == int(c), f"E2M1 code of {v}: {got}, expected {c}"
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    # every code decodes to its grid value and encodes back to itself
    for c in range(16):
        val = float(decode(np.array([c]))[0])
        mag = grid[c & 7]
        assert val == (-mag if c & 8 else mag), f"E2M1 decode of {c}"
        assert int(encode(np.array([val]))[0]) == (c if mag != 0 or c == 0 else 8), f"E2M1 round trip of {c}"
    # brute force on a fine grid: nearest grid value, a tie to the even code, saturation at 6
    t = np.arange(-8 * 64, 8 * 64 + 1) / 64.0
    codes = encode(t).astype(np.int64)
    for x, c in zip(t, codes):
        d = np.abs(grid - min(abs(x), 6.0))
        near = np.flatnonzero(d == d.min())
        want = near[0] if len(near) == 1 else near[near % 2 == 0][0]
        assert (c & 7) == want, f"E2M1 rounding of {x}"
        assert (c >> 3) == (1 if x < 0 else 0), f"E2M1 sign of {x}"


def check_e4m3(encode, decode):
    import torch
    for row in _golden_rows("nvfp4_e4m3_examples.txt"):
        v, c = (p.strip() for p in row.split("|"))
        got = int(encode(np.array([float(v)]))[0])
        assert got == int(c, 16), f"E4M3 code of {v}: {got:#x}, expected 0x{c}"
    codes = np.arange(127)
    vals = decode(codes)
    assert np.all(np.diff(vals) > 0), "E4M3 values must rise with the code"
    assert np.array_equal(encode(vals).astype(np.int64), codes), "E4M3 round trip"
    # an independent reference: PyTorch's float8_e4m3fn cast (round to nearest even) on the
    # finite range, and on the decoded values themselves
    ref_vals = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(vals, ref_vals), "E4M3 values differ from PyTorch's float8_e4m3fn"
    rng = np.random.default_rng(17)
    s = np.concatenate([rng.uniform(0, 448, 4000), 2.0 ** rng.uniform(-12, 8.8, 4000), (vals[1:] + vals[:-1]) / 2])
    s = np.minimum(s, 448.0).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(s.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(encode(s).astype(np.uint8), ref), "E4M3 rounding differs from PyTorch's cast"
    assert int(encode(np.array([1e6]))[0]) == 0x7E, "E4M3 must saturate at 448"


def check_nvfp4_quantizer(quantize):
    for row in _golden_rows("nvfp4_quant_examples.txt"):
        z_s, c_s, s_s, sx_s = (p.strip() for p in row.split("|"))
        z = np.array([[float(v) for v in z_s.split()]], dtype=np.float32)
        codes, sb, s_x = quantize(z, 64)
        assert np.array_equal(codes[0].astype(np.int64), [int(v) for v in c_s.split()]), f"NVFP4 codes of {z_s[:40]}"
        assert np.array_equal(sb[0].astype(np.int64), [int(v, 16) for v in s_s.split()]), "NVFP4 block scales"
        assert s_x[0] == float(sx_s), "NVFP4 token scale"
    import oracle
    rng = np.random.default_rng(19)
    z = (rng.standard_normal((40, 256)) * rng.uniform(0.01, 100, size=(40, 1))).astype(np.float32)
    z[:, 32:48] *= 1e-3            # a quiet block
    z[5] = 0.0
    codes, sb, s_x = quantize(z, 64)
    e = oracle.e2m1_decode(codes)
    s = np.repeat(oracle.e4m3_decode(sb), 16, axis=1)
    a = np.abs(z).max(1).astype(np.float64)
    live = a > 0
    assert not np.any(codes[5] & 7) and s_x[5] == 0.0, "zero row"
    # reconstruction: u / sb within half the local E2M1 spacing (plus the scale's own rounding)
    u = z.astype(np.float64) * (2688.0 / np.where(live, a, 1.0))[:, None]
    t = np.divide(u, s, out=np.zeros_like(u), where=s > 0)
    spacing = np.where(np.abs(t) < 2, 0.5, np.where(np.abs(t) < 4, 1.0, 2.0))
    ok = np.abs(e - np.clip(t, -6, 6)) <= 0.5 * spacing + 1e-6
    assert np.all(ok[live]), "codes further than half a step from u / sb"
    # each block's largest |u| lands at the top of the E2M1 range (4 or 6: the scale rounds)
    top = np.abs(e).reshape(40, 16, 16).max(2)
    assert np.all(top[live][sb[live] > 0] >= 4.0), "block absmax does not use the top of the range"
    # the token's absmax block gets the largest scale, 448 (E4M3 0x7E)
    assert np.all(sb[live].max(1) == 0x7E)
    assert np.allclose(s_x[live], a[live] / (2688 * 8.0), rtol=1e-15)
    # sign symmetry (zeros keep their own sign)
    cn, sbn, _ = quantize(-z, 64)
    assert np.array_equal(sbn, sb) and np.array_equal(cn & 7, codes & 7), "NVFP4 quantizer is not symmetric"


def check_nvfp4_weights(quantize_w):
    for row in _golden_rows("nvfp4_weight_examples.txt"):
        w_s, c_s, s_s = (p.strip() for p in row.split("|"))
        w = np.array([[int(v) for v in w_s.split()]], dtype=np.int8)
        codes, sb = quantize_w(w)
        assert np.array_equal(codes[0].astype(np.int64), [int(v) for v in c_s.split()]), "NVFP4 weight codes"
        assert int(sb[0, 0]) == int(s_s, 16), "NVFP4 weight block scale"


def check_nvfp4_gemm(gemm):
    from fractions import Fraction
    import oracle
    rng = np.random.default_rng(23)
    for (M, N, K) in ((1, 1, 16), (2, 3, 32), (3, 2, 64)):
        ca = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
        cw = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
        sa = rng.integers(0, 127, size=(M, K // 16)).astype(np.uint8)
        sw = rng.integers(0, 127, size=(N, K // 16)).astype(np.uint8)
        acc = gemm(ca, sa, cw, sw)

        def val_e2m1(c):
            mag = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)][c & 7]
            return -mag if c & 8 else mag

        def val_e4m3(c):
            e, m = c >> 3, c & 7
            return Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)

        for i in range(M):
            for j in range(N):
                exact = sum(val_e2m1(int(ca[i, k])) * val_e4m3(int(sa[i, k // 16])) *
                            val_e2m1(int(cw[j, k])) * val_e4m3(int(sw[j, k // 16])) for k in range(K))
                assert Fraction(float(acc[i, j])) == exact, f"NVFP4 GEMM ({i}, {j}) != exact sum"
