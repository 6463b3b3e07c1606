"""The on-device DMPQ precision predictor (tasq_dmpq_update) against the oracle.

Gamma = ||out - in||_1 / ||in||_1 of a block at the previous step picks the bit width of the
block's linears for the next step (6Bit-Diffusion section 2.A, DMPQ). Both sides take the two
L1 sums exactly and divide in IEEE double, so Gamma must agree bit for bit and the decision
must match, even with tau set exactly at Gamma.
"""
import math

import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

F16_REL = 1e-3
ABS_TINY = 2.0 ** -24


@pytest.fixture(scope="module")
def T():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from conftest import build_library
    return build_library()


def _s():
    return torch.cuda.current_stream()


def _pair(rng, M, D, ld_extra=0, scale=3.0):
    x_in = (rng.standard_normal((M, D)) * scale).astype(np.float32)
    cols = rng.choice(D, size=max(1, D // 200), replace=False)
    x_in[:, cols] *= 50
    x_out = x_in + (rng.standard_normal((M, D)) * scale * rng.uniform(0.01, 1.0)).astype(np.float32)
    x_in, x_out = x_in.astype(np.float16), x_out.astype(np.float16)
    ld = D + ld_extra
    din = np.zeros((M, ld), np.float16)
    dout = np.zeros((M, ld), np.float16)
    din[:, :D] = x_in
    dout[:, :D] = x_out
    return x_in, x_out, torch.from_numpy(din).cuda(), torch.from_numpy(dout).cuda(), ld


def _ctx(T, num_layers, steps):
    layers = [(64, 64, np.zeros((64, 64), np.int8), np.ones(64, np.float32)) for _ in range(num_layers)]
    return T.tasq_linear_create(layers, steps, 64, 16, T.TASQ_OUT_F16, _s())


@pytest.mark.parametrize("M,D,ld_extra", [(1, 8, 0), (3, 24, 8), (257, 1152, 0), (1000, 2240, 16),
                                          (4096, 3072, 0), (8192, 1152, 8)])
def test_gamma_and_bits_match_oracle(T, M, D, ld_extra):
    rng = np.random.default_rng(M * 3 + D)
    x_in, x_out, din, dout, ld = _pair(rng, M, D, ld_extra)
    ctx = _ctx(T, 6, 5)
    before = T.tasq_get_schedule(ctx, _s())
    g = torch.full((1,), float("nan"), dtype=torch.float64, device="cuda")
    want = oracle.dmpq_gamma(x_in, x_out)
    tau = 0.3
    T.tasq_dmpq_update(ctx, din, ld, dout, ld, M, D, [1, 4, 5], 2, tau, 8, 4, g, _s())
    got = float(g.item())
    assert got == want, f"Gamma {got!r} vs oracle {want!r}"
    table = T.tasq_get_schedule(ctx, _s())
    bits = oracle.dmpq_bits(want, tau, 8, 4)
    expect = before.copy()
    expect[[1, 4, 5], 2] = bits
    assert np.array_equal(table, expect), "only the listed (layer, step) entries change"
    assert T.tasq_get_device_status(ctx) == 0


def test_decision_at_the_threshold(T):
    rng = np.random.default_rng(5)
    x_in, x_out, din, dout, ld = _pair(rng, 300, 640)
    gamma = oracle.dmpq_gamma(x_in, x_out)
    ctx = _ctx(T, 2, 3)
    # tau exactly Gamma: Gamma > tau is false, so stable; one ulp below: unstable
    T.tasq_dmpq_update(ctx, din, ld, dout, ld, 300, 640, [0], 0, gamma, 8, 3, None, _s())
    T.tasq_dmpq_update(ctx, din, ld, dout, ld, 300, 640, [1], 0, math.nextafter(gamma, -math.inf), 7, 3, None, _s())
    table = T.tasq_get_schedule(ctx, _s())
    assert table[0, 0] == 3 and table[1, 0] == 7


def test_zero_input_and_extremes(T):
    ctx = _ctx(T, 3, 2)
    g = torch.zeros((1,), dtype=torch.float64, device="cuda")
    z = torch.zeros((4, 16), dtype=torch.float16, device="cuda")
    # no input magnitude, no change: Gamma 0, no information, the wide width
    T.tasq_dmpq_update(ctx, z, 16, z, 16, 4, 16, [0], 1, 0.5, 8, 4, g, _s())
    assert float(g.item()) == 0.0
    one = z.clone()
    one[2, 3] = 1.0
    T.tasq_dmpq_update(ctx, z, 16, one, 16, 4, 16, [1], 1, 1e300, 6, 4, g, _s())
    assert math.isinf(float(g.item()))
    # largest FP16 magnitudes and subnormals: the exact sums span 2^-24 .. 2^41 units per element
    big = np.full((64, 64), 65504, np.float16)
    big[::2] = -65504
    big[1, :8] = np.float16(2.0 ** -24)
    T.tasq_dmpq_update(ctx, torch.from_numpy(big).cuda(), 64, torch.from_numpy(-big).cuda(), 64, 64, 64, [2], 1,
                       1.9, 8, 4, g, _s())
    assert float(g.item()) == oracle.dmpq_gamma(big, -big) == 2.0
    table = T.tasq_get_schedule(ctx, _s())
    assert table[0, 1] == 8 and table[1, 1] == 6 and table[2, 1] == 8


def _all_finite_fp16(rng, max_exponent_field=30):
    """Every finite FP16 bit pattern whose exponent field is at most max_exponent_field (both
    signs, both zeros), in random order."""
    h = np.arange(65536, dtype=np.uint32)
    h = h[((h >> 10) & 31) <= max_exponent_field]
    return rng.permutation(h).astype(np.uint16).view(np.float16)


def test_every_finite_fp16_value_enters_the_sums_exactly(T):
    """Input and output each hold every finite FP16 value once (63488 patterns as 248 x 256), in
    two different orders; then only subnormals and the smallest normals (|x| < 2^-11, 8192
    patterns), where both sums stay below 2^53 units: Gamma is then the quotient of two exact
    doubles, and one unit more or less in either sum changes it."""
    rng = np.random.default_rng(17)
    ctx = _ctx(T, 2, 1)
    g = torch.zeros((1,), dtype=torch.float64, device="cuda")
    for idx, (max_e, M, D) in enumerate([(30, 248, 256), (3, 32, 256)]):
        x_in = _all_finite_fp16(rng, max_e).reshape(M, D)
        x_out = _all_finite_fp16(rng, max_e).reshape(M, D)
        T.tasq_dmpq_update(ctx, torch.from_numpy(x_in).cuda(), D, torch.from_numpy(x_out).cuda(), D, M, D, [idx],
                           0, 0.5, 8, 4, g, _s())
        num, den = oracle.dmpq_l1_sums(x_in, x_out)
        if max_e == 3:
            assert num < 2 ** 53 and den < 2 ** 53
            assert float(num + 1) / float(den) != float(num) / float(den)
        assert float(g.item()) == oracle.dmpq_gamma(x_in, x_out), max_e
    assert T.tasq_get_device_status(ctx) == 0


def test_full_size_sums_stay_exact(T):
    """CogVideoX-sized block (17776 x 3072) at the largest magnitudes: the exact sums exceed 2^64
    units, which the 128-bit partial sums must carry."""
    M, D = 17776, 3072
    rng = np.random.default_rng(11)
    x_in = np.where(rng.random((M, D)) < 0.5, np.float16(65504), np.float16(-65504)).astype(np.float16)
    x_out = (-x_in).astype(np.float16)
    x_out[rng.random((M, D)) < 0.1] = np.float16(0.0)
    ctx = _ctx(T, 1, 1)
    g = torch.zeros((1,), dtype=torch.float64, device="cuda")
    T.tasq_dmpq_update(ctx, torch.from_numpy(x_in).cuda(), D, torch.from_numpy(x_out).cuda(), D, M, D, [0], 0, 1.5,
                       8, 4, g, _s())
    num, den = oracle.dmpq_l1_sums(x_in, x_out)
    assert den > 2 ** 64
    assert float(g.item()) == oracle.dmpq_gamma(x_in, x_out)


def test_new_widths_apply_to_the_next_forward_in_stream_order(T):
    """Predictor then forward on one stream, no synchronisation in between: the forward uses the
    width the predictor just wrote."""
    rng = np.random.default_rng(21)
    M, K, N, n = 256, 1152, 1152, 64
    x = (rng.standard_normal((M, K))).astype(np.float16)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    ctx = T.tasq_linear_create([(N, K, w, s_w)], 2, n, M, T.TASQ_OUT_F16, _s())
    x_in, x_out, din, dout, ld = _pair(rng, M, K)
    gamma = oracle.dmpq_gamma(x_in, x_out)
    xd = torch.from_numpy(x).cuda()
    ys = []
    for step, tau in ((0, gamma * 2), (1, gamma / 2)):      # stable, then unstable
        T.tasq_dmpq_update(ctx, din, ld, dout, ld, M, K, [0], step, tau, 8, 3, None, _s())
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        T.tasq_linear_forward(ctx, xd, M, K, 0, step, y, N, _s())
        ys.append(y)
    torch.cuda.synchronize()
    for y, bits in zip(ys, (3, 8)):
        ref = oracle.masked_linear(x, w, s_w, bits, n)["y"]
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY), f"bits={bits}"
    assert T.tasq_get_device_status(ctx) == 0


def test_argument_errors(T):
    ctx = _ctx(T, 2, 2)
    z = torch.zeros((4, 32), dtype=torch.float16, device="cuda")

    def err(*a):
        with pytest.raises(T.TasqError) as ei:
            T.tasq_dmpq_update(ctx, *a)
        return ei.value.status

    E = T.TASQ_ERR_INVALID_ARG
    assert err(z, 32, z, 32, 4, 12, [0], 0, 0.5, 8, 4, None, _s()) == E          # D % 8
    assert err(z, 32, z, 32, 4, 32, [], 0, 0.5, 8, 4, None, _s()) == E           # no layers
    assert err(z, 32, z, 32, 4, 32, [0] * 33, 0, 0.5, 8, 4, None, _s()) == E     # too many
    assert err(z, 32, z, 32, 4, 32, [2], 0, 0.5, 8, 4, None, _s()) == E          # layer range
    assert err(z, 32, z, 32, 4, 32, [0], 2, 0.5, 8, 4, None, _s()) == E          # step range
    assert err(z, 32, z, 32, 4, 32, [0], 0, 0.5, 9, 4, None, _s()) == E          # bits
    assert err(z, 32, z, 32, 4, 32, [0], 0, 0.5, 8, -1, None, _s()) == E         # bits
    assert err(z, 32, z, 32, 4, 32, [0], 0, float("nan"), 8, 4, None, _s()) == E
    assert err(z.data_ptr() + 2, 32, z, 32, 4, 32, [0], 0, 0.5, 8, 4, None, _s()) == E   # alignment
    assert err(z, 30, z, 32, 4, 32, [0], 0, 0.5, 8, 4, None, _s()) == E          # row stride
    assert np.all(T.tasq_get_schedule(ctx, _s()) == 8), "a rejected call changes nothing"


def _nvfp4_close(got, x, w, s_w, n):
    r = oracle.nvfp4_linear(x, w, s_w, n)
    Kp = oracle.padded_k(x.shape[1], n)
    bound = (Kp * 2.0 ** -24 * oracle.nvfp4_abs_terms(r["ca"], r["sa"], r["cw"], r["sw"]) * 1.0001 *
             r["s_x"][:, None] * s_w[None, :] + np.abs(r["y"]) * (2.0 ** -11 + 2.0 ** -21) + 2.0 ** -24)
    return np.all(np.abs(got - r["y"]) <= bound)


def test_predictor_chooses_int8_or_nvfp4_on_the_device(T):
    """6Bit-Diffusion's split: unstable blocks INT8, stable ones NVFP4, decided on the device. The
    forward after the predictor launches both paths gated on the table; the output is the INT8
    result when Gamma > tau and the NVFP4 result otherwise, with no host round trip, also from a
    CUDA graph captured once and replayed after the decision changed."""
    rng = np.random.default_rng(23)
    M, K, N, n = 384, 1152, 896, 64
    x = (rng.standard_normal((M, K))).astype(np.float16)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    ctx = T.tasq_linear_create([(N, K, w, s_w)], 1, n, M, T.TASQ_OUT_F16, _s())
    x_in, x_out, din, dout, ld = _pair(rng, M, K)
    gamma = oracle.dmpq_gamma(x_in, x_out)
    xd = torch.from_numpy(x).cuda()
    ref8 = oracle.masked_linear(x, w, s_w, 8, n)["y"]
    # direct launches: stable -> NVFP4, then unstable -> INT8
    for tau, want in ((gamma * 2, "nvfp4"), (gamma / 2, "int8")):
        T.tasq_dmpq_update(ctx, din, ld, dout, ld, M, K, [0], 0, tau, 8, T.TASQ_NVFP4, None, _s())
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        T.tasq_linear_forward(ctx, xd, M, K, 0, 0, y, N, _s())
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        assert int(T.tasq_get_schedule(ctx, _s())[0, 0]) == (0 if want == "nvfp4" else 8)
        if want == "nvfp4":
            assert _nvfp4_close(got, x, w, s_w, n), "NVFP4 chosen on the device"
        else:
            assert np.all(np.abs(got - ref8) <= F16_REL * np.abs(ref8) + ABS_TINY), "INT8 chosen on the device"
    # one captured graph of predictor + forward, replayed with tau moved between replays
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    T.tasq_dmpq_update(ctx, din, ld, dout, ld, M, K, [0], 0, gamma * 2, 8, T.TASQ_NVFP4, None, _s())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        T.tasq_linear_forward(ctx, xd, M, K, 0, 0, y, N, torch.cuda.current_stream())
    for tau, want in ((gamma * 2, "nvfp4"), (gamma / 2, "int8"), (gamma * 2, "nvfp4")):
        T.tasq_dmpq_update(ctx, din, ld, dout, ld, M, K, [0], 0, tau, 8, T.TASQ_NVFP4, None, _s())
        g.replay()
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        if want == "nvfp4":
            assert _nvfp4_close(got, x, w, s_w, n), "graph replay, NVFP4"
        else:
            assert np.all(np.abs(got - ref8) <= F16_REL * np.abs(ref8) + ABS_TINY), "graph replay, INT8"
    assert T.tasq_get_device_status(ctx) == 0
