"""The oracle against what the pages and the mathematics fix (CPU only)."""
import math

import numpy as np
import pytest

import oracle
import pins
import workloads


def test_hadamard_matrix():
    pins.check_hadamard_matrix(oracle.sylvester_hadamard)


def test_block_hadamard_exact():
    pins.check_block_hadamard_exact(oracle.block_hadamard_exact)


def test_block_hadamard_fp32():
    pins.check_block_hadamard_fp32(oracle.block_hadamard_fp32, oracle.block_hadamard_exact)


def test_quantizer():
    pins.check_quantizer(oracle.quantize_per_token)


def test_mask():
    pins.check_mask(oracle.lsb_mask)


def test_gemm():
    pins.check_gemm(oracle.int_gemm)


def test_dequant():
    pins.check_dequant(oracle.dequant)


def test_end_to_end():
    pins.check_end_to_end(oracle.masked_linear, oracle.block_hadamard_exact, oracle.sylvester_hadamard)


def test_fp32_codes_track_exact_codes():
    """Codes decided on the FP32 transform differ from codes decided on the exact transform by
    at most one step, and rarely (the tolerance the method states is 0.1 % of codes)."""
    wl = workloads.WORKLOADS["single"]
    x = workloads.activations(wl, 0)
    q32, _, _ = oracle.prologue(x, wl.hadamard_n)
    z64 = oracle.block_hadamard_exact(x, wl.hadamard_n)
    a = np.abs(z64).max(1)
    q64 = np.clip(np.rint(z64 * (127.0 / a)[:, None]), -127, 127).astype(np.int64)
    d = np.abs(q32.astype(np.int64) - q64)
    assert d.max() <= 1
    assert d.astype(bool).mean() <= 1e-3


def test_bitops_model():
    # TASQ: bit-serial cycles scale with w_bits * a_bits
    assert oracle.bitops(2, 3, 4, 8, 8) == 2 * 3 * 4 * 64
    assert oracle.bitops(256, 1152, 1152, 4) * 2 == oracle.bitops(256, 1152, 1152, 8)


def test_masked_linear_shapes_and_ranges():
    wl = workloads.WORKLOADS["single"]
    x = workloads.activations(wl, 0, M=40)
    w, s_w = workloads.weights(wl, 0)
    out = oracle.masked_linear(x, w, s_w, 5, wl.hadamard_n)
    assert out["q"].shape == (40, 1152) and out["q"].dtype == np.int8
    assert out["acc"].shape == (40, 1152)
    assert np.all(np.abs(out["acc"]) < 2 ** 31)
    assert np.all(np.isfinite(out["y"]))
    assert np.all(out["wk"].astype(np.int64) % 8 == 0)


@pytest.mark.parametrize("name", workloads.WORKLOAD_ORDER)
def test_outputs_fit_fp16(name):
    """The workloads' outputs stay inside the FP16 range (checked on a row sample of every
    distinct layer shape at bits = 8, the largest-magnitude case)."""
    wl = workloads.WORKLOADS[name]
    seen = set()
    for layer in range(len(wl.block_layers)):
        _, K, N = wl.layer_shape(layer)
        if (K, N) in seen:
            continue
        seen.add((K, N))
        x = workloads.activations(wl, layer, M=min(wl.tokens, 48))
        w, s_w = workloads.weights(wl, layer)
        y = oracle.masked_linear(x, w, s_w, 8, wl.hadamard_n)["y"]
        assert np.abs(y).max() < 65504 / 4


def test_dmpq_predictor():
    pins.check_dmpq(oracle.dmpq_gamma, oracle.dmpq_bits, oracle.dmpq_l1_sums)


def test_nvfp4_e2m1():
    pins.check_e2m1(oracle.e2m1_encode, oracle.e2m1_decode)


def test_nvfp4_e4m3():
    pins.check_e4m3(oracle.e4m3_encode, oracle.e4m3_decode)


def test_nvfp4_quantizer():
    pins.check_nvfp4_quantizer(oracle.nvfp4_quantize_activations)


def test_nvfp4_weights():
    pins.check_nvfp4_weights(oracle.nvfp4_quantize_weights)


def test_nvfp4_gemm():
    pins.check_nvfp4_gemm(oracle.nvfp4_gemm)


def test_nvfp4_linear_approximates_the_real_product():
    """End-to-end algebra: with the stored weights in the rotated basis (R3), y ~= x W_real^T,
    W_real = s_w * W H_blk / sqrt(n), within the NVFP4 quantization error (a sanity check)."""
    rng = np.random.default_rng(29)
    M, N, K, n = 8, 12, 128, 64
    x = rng.standard_normal((M, K)).astype(np.float16)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N)
    r = oracle.nvfp4_linear(x, w, s_w, n)
    H = oracle.sylvester_hadamard(n).astype(np.float64)
    Hb = np.kron(np.eye(K // n), H)
    y_real = x.astype(np.float64) @ (w.astype(np.float64) * s_w[:, None] @ Hb / math.sqrt(n)).T
    rel = np.linalg.norm(r["y"] - y_real) / np.linalg.norm(y_real)
    assert rel < 0.2, f"NVFP4 W4A4 relative error {rel}"
