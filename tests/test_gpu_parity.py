"""CUDA path against the CPU oracle, element by element, through the C ABI.

Bars (from the method's stated tolerances):
  * INT32 accumulators: bit-exact.
  * INT8 activation codes: at most 0.1 % differ, none by more than 1 (both sides decide them in
    FP32 with the same butterfly order, so they are expected to agree exactly).
  * s_x: relative error <= 1e-6 (FP32 scale against the FP64 definition).
  * FP16 outputs given identical codes: |dy| <= 1e-3 |y| + 2^-24 elementwise;
    BF16 outputs: |dy| <= 2^-8 |y| + 2^-24 (one BF16 rounding of an FP32 product).
  * Whole forward: ||dy||_F / ||y||_F <= 1e-3.
"""
import math

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

F16_REL = 1e-3
ABS_TINY = 2.0 ** -24


@pytest.fixture(scope="module")
def T():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from conftest import build_library
    t = build_library()
    torch.cuda.init()
    return t


def _stream():
    return torch.cuda.current_stream()


def _acts(rng, M, K, outliers=True):
    x = rng.standard_normal((M, K), dtype=np.float32)
    if outliers:
        cols = rng.choice(K, size=max(1, K // 200), replace=False)
        x[:, cols] *= 50
    return x.astype(np.float16)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _codes_ok(q_gpu, q_ref):
    d = np.abs(q_gpu.astype(np.int64) - q_ref.astype(np.int64))
    assert d.max(initial=0) <= 1, f"a code differs by {d.max()}"
    frac = d.astype(bool).mean() if d.size else 0.0
    assert frac <= 1e-3, f"{frac:.2e} of codes differ"
    return frac


def _ctx(T, layers, steps, n, max_tokens, out=0):
    return T.tasq_linear_create(layers, steps, n, max_tokens, out, _stream())


# ----------------------------------------------------------------------------- prologue
# prologue kernels: 1 = direct loads (32 channels a thread), 2 = bulk-fed ring wherever its layout
# fits, 3 = direct loads with 64 channels a thread
@pytest.mark.parametrize("pmode", [1, 2, 3])
@pytest.mark.parametrize("n,K,M", [(64, 64, 1), (64, 96, 3), (64, 1152, 257), (128, 2240, 130), (128, 128, 5),
                                   (64, 12288, 33), (128, 16384, 2), (64, 4608, 300), (128, 5600, 64),
                                   (64, 1152, 4000), (64, 640, 9001), (128, 3072, 1500)])
def test_prologue_matches_oracle(T, n, K, M, pmode):
    rng = np.random.default_rng(K * 31 + M)
    x = _acts(rng, M, K)
    if M >= 3:
        x[1] = 0                    # all-zero token: codes 0, scale 0
        x[2] = np.float16(0.5)      # constant token
    Kp = oracle.padded_k(K, n)
    ctx = _ctx(T, [(64, K, np.zeros((64, Kp), np.int8), np.ones(64, np.float32))], 1, n, max(M, 1))
    T.tasq_debug_set_prologue_mode(ctx, pmode)
    ldx = K + 8                     # strided rows
    xs = np.zeros((M, ldx), np.float16)
    xs[:, :K] = x
    xd = _dev(xs)
    # codes 16-byte but not 32-byte aligned for odd M: the narrower store path
    off = 16 if M % 2 == 1 else 0
    xq_buf = torch.empty((M * Kp + 64,), dtype=torch.int8, device="cuda")
    xq = xq_buf[off:off + M * Kp].view(M, Kp)
    sx = torch.empty((M,), dtype=torch.float32, device="cuda")
    T.tasq_debug_quantize(ctx, xd, M, ldx, 0, xq, sx, _stream())
    torch.cuda.synchronize()
    q_ref, sx_ref, _ = oracle.prologue(x, n)
    frac = _codes_ok(xq.cpu().numpy(), q_ref)
    assert frac == 0.0, "codes are decided in FP32 in the same butterfly order on both sides"
    sx_g = sx.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(sx_g - sx_ref) <= 1e-6 * np.abs(sx_ref)), "s_x"
    if M >= 3:
        assert sx_g[1] == 0.0 and not xq[1].any().item()
    assert T.tasq_get_device_status(ctx) == 0


# rows whose transform is exact and whose scaled values are exact ties: z = blockwise x H_n holds
# 254 once and small odd integers elsewhere, so a = 254, fp32(127 / a) = 0.5 and every other
# z * 0.5 is a half-integer. x = z H_n / n is a multiple of 1/n below 2^11 / n, exact in FP16, and
# every butterfly sum of it is exact in FP32, so both sides see the same exact ties.
@pytest.mark.parametrize("pmode", [1, 2, 3])
@pytest.mark.parametrize("n,blocks,M", [(64, 3, 37), (128, 2, 20), (64, 18, 600)])
def test_prologue_exact_ties_round_to_even(T, n, blocks, M, pmode):
    rng = np.random.default_rng(n * 1000 + blocks * 10 + M)
    K = n * blocks
    z = (2 * rng.integers(-3, 4, size=(M, K)) + 1).astype(np.float64)   # odd, |z| <= 7
    z[np.arange(M), rng.integers(0, K, size=M)] = 254.0
    H = oracle.sylvester_hadamard(n).astype(np.float64)
    x = np.concatenate([z[:, b * n:(b + 1) * n] @ H / n for b in range(blocks)], axis=1)
    assert np.array_equal(x.astype(np.float16).astype(np.float64), x)
    x = x.astype(np.float16)
    ctx = _ctx(T, [(64, K, np.zeros((64, K), np.int8), np.ones(64, np.float32))], 1, n, M)
    T.tasq_debug_set_prologue_mode(ctx, pmode)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty((M,), dtype=torch.float32, device="cuda")
    T.tasq_debug_quantize(ctx, _dev(x), M, K, 0, xq, sx, _stream())
    torch.cuda.synchronize()
    q_ref, sx_ref, _ = oracle.prologue(x, n)
    assert np.array_equal(q_ref, np.rint(z / 2.0).astype(np.int8)), "oracle: ties to even"
    assert np.array_equal(xq.cpu().numpy(), q_ref), "ties must round to even on the GPU too"
    assert np.all(np.abs(sx.cpu().numpy().astype(np.float64) - sx_ref) <= 1e-6 * sx_ref)


# ----------------------------------------------------------------------------- GEMM, exact
# (GEMM kernel, mask placement): kernel 1 = one CTA per 128 x 256 tile, 2 = CTA pairs on
# 256 x 256 tiles; placement 1 = every weight tile masked in shared memory inside the GEMM,
# 2 = the layer's weights masked once ahead of the GEMM in the prologue launch
GEMM_MODES = [(1, 1), (1, 2), (2, 1), (2, 2)]


def _set_modes(T, ctx, mode):
    gemm, mask = mode
    T.tasq_debug_set_gemm_mode(ctx, gemm)
    T.tasq_debug_set_mask_mode(ctx, mask)


@pytest.mark.parametrize("mode", GEMM_MODES)
@pytest.mark.parametrize("M,N,K,n", [(1, 1, 64, 64), (256, 128, 128, 64), (300, 200, 1152, 64), (513, 384, 192, 64),
                                     (100, 1152, 2240, 128), (257, 130, 4608, 64), (64, 2000, 64, 64),
                                     (700, 520, 320, 64), (576, 256, 1152, 64)])
def test_gemm_s32_bit_exact_all_bits(T, M, N, K, n, mode):
    rng = np.random.default_rng(M * 7 + N * 13 + K)
    Kp = oracle.padded_k(K, n)
    w = rng.integers(-128, 128, size=(N, Kp)).astype(np.int8)     # includes -128
    q = rng.integers(-127, 128, size=(M, Kp)).astype(np.int8)
    steps = 8
    ctx = _ctx(T, [(N, K, w, np.ones(N, np.float32))], steps, n, M)
    _set_modes(T, ctx, mode)
    bits = np.array([[8, 7, 6, 5, 4, 3, 2, 1]], np.uint8)
    T.tasq_set_schedule(ctx, bits, _stream())
    qd = _dev(q)
    ld = N + (8 - N % 8) % 8 + 8
    for step in range(steps):
        acc = torch.full((M, ld), 0x7F7F7F7F, dtype=torch.int32, device="cuda")
        T.tasq_debug_gemm_s32(ctx, qd, M, 0, step, acc, ld, _stream())
        torch.cuda.synchronize()
        got = acc.cpu().numpy()
        ref = oracle.int_gemm(q, oracle.lsb_mask(w, int(bits[0, step])))
        assert np.array_equal(got[:, :N].astype(np.int64), ref), f"INT32 accumulators differ at bits={bits[0, step]}"
        assert np.all(got[:, N:] == 0x7F7F7F7F), "write outside [M, N]"
    assert T.tasq_get_device_status(ctx) == 0


@pytest.mark.parametrize("mode", GEMM_MODES)
def test_gemm_extreme_values(T, mode):
    """All-(-128) weights at k = 0 and all-(-127) codes: the largest accumulators at Kp = 12288."""
    M, N, K = 256, 128, 12288
    w = np.full((N, K), -128, np.int8)
    w[::2] = 127
    q = np.full((M, K), -127, np.int8)
    q[::3] = 127
    ctx = _ctx(T, [(N, K, w, np.ones(N, np.float32))], 2, 64, M)
    _set_modes(T, ctx, mode)
    T.tasq_set_schedule(ctx, np.array([[8, 1]], np.uint8), _stream())
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    for step, bits in ((0, 8), (1, 1)):
        T.tasq_debug_gemm_s32(ctx, _dev(q), M, 0, step, acc, N, _stream())
        torch.cuda.synchronize()
        ref = oracle.int_gemm(q, oracle.lsb_mask(w, bits))
        assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)


# ----------------------------------------------------------------------------- dequant epilogue
@pytest.mark.parametrize("mode", GEMM_MODES)
@pytest.mark.parametrize("out", [0, 1])
@pytest.mark.parametrize("M,N,K", [(300, 200, 1152), (17, 1152, 64), (512, 256, 256)])
def test_gemm_dequant_given_codes(T, out, M, N, K, mode):
    rng = np.random.default_rng(M + N + K + out)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    s_x = rng.uniform(0.01, 3.0, size=M).astype(np.float32)
    s_x[0] = 0.0
    ctx = _ctx(T, [(N, K, w, s_w)], 2, 64, M)
    _set_modes(T, ctx, mode)
    T.tasq_set_schedule(ctx, np.array([[8, 5]], np.uint8), _stream())
    tdt = torch.float16 if out == 0 else torch.bfloat16
    for step, bits in ((0, 8), (1, 5)):
        y = torch.full((M, N), float("nan"), dtype=tdt, device="cuda")
        T.tasq_debug_gemm(ctx, _dev(q), _dev(s_x), M, 0, step, y, N, out, _stream())
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        ref = oracle.dequant(oracle.int_gemm(q, oracle.lsb_mask(w, bits)), s_x, s_w)
        rel = F16_REL if out == 0 else 2.0 ** -8
        assert np.all(np.abs(got - ref) <= rel * np.abs(ref) + ABS_TINY), "dequantized outputs"


# ----------------------------------------------------------------------------- whole forward
@pytest.mark.parametrize("mode", [(0, 0)] + GEMM_MODES)
@pytest.mark.parametrize("n,K,N,M", [(64, 1152, 1152, 256), (64, 1152, 3456, 300), (128, 2240, 6720, 130),
                                     (64, 4608, 1152, 77), (128, 5600, 2240, 513), (64, 64, 8, 1)])
def test_forward_matches_oracle(T, n, K, N, M, mode):
    rng = np.random.default_rng(n + K + N + M)
    Kp = oracle.padded_k(K, n)
    x = _acts(rng, M, K)
    w = rng.integers(-127, 128, size=(N, Kp)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    bits_per_step = [8, 6, 5, 4, 3]
    ctx = _ctx(T, [(N, K, w, s_w)], len(bits_per_step), n, M + 5)
    _set_modes(T, ctx, mode)
    T.tasq_set_schedule(ctx, np.array([bits_per_step], np.uint8), _stream())
    xd = _dev(x)
    ldy = N + (8 - N % 8) % 8 + 16
    ref_q, ref_sx, _ = oracle.prologue(x, n)
    for step, bits in enumerate(bits_per_step):
        y = torch.full((M + 2, ldy), float("nan"), dtype=torch.float16, device="cuda")
        T.tasq_linear_forward(ctx, xd, M, K, 0, step, y, ldy, _stream())
        torch.cuda.synchronize()
        got_all = y.float().cpu().numpy()
        assert np.isnan(got_all[:M, N:]).all() and np.isnan(got_all[M:]).all(), "write outside [M, N]"
        got = got_all[:M, :N].astype(np.float64)
        ref = oracle.masked_linear(x, w, s_w, bits, n)["y"]
        assert np.linalg.norm(got - ref) <= 1e-3 * np.linalg.norm(ref)
        assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY), "elementwise (codes agree exactly)"
    assert T.tasq_get_device_status(ctx) == 0


@pytest.mark.parametrize("n,K,N,M", [(64, 1152, 1152, 300), (128, 5600, 2240, 513), (64, 4608, 640, 2000)])
def test_forward_bulk_fed_prologue_with_weight_pass(T, n, K, N, M):
    """The bulk-fed prologue on a whole forward, with the weights masked ahead by the same
    persistent CTAs after their rows (every step drops bits)."""
    rng = np.random.default_rng(n + K + N + M + 7)
    Kp = oracle.padded_k(K, n)
    x = _acts(rng, M, K)
    w = rng.integers(-128, 128, size=(N, Kp)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    bits_per_step = [7, 4, 1]
    ctx = _ctx(T, [(N, K, w, s_w)], len(bits_per_step), n, M)
    T.tasq_debug_set_prologue_mode(ctx, 2)
    T.tasq_debug_set_mask_mode(ctx, 2)
    T.tasq_set_schedule(ctx, np.array([bits_per_step], np.uint8), _stream())
    xd = _dev(x)
    for step, bits in enumerate(bits_per_step):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        T.tasq_linear_forward(ctx, xd, M, K, 0, step, y, N, _stream())
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        ref = oracle.masked_linear(x, w, s_w, bits, n)["y"]
        assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY), f"bits={bits}"
    assert T.tasq_get_device_status(ctx) == 0


@pytest.mark.parametrize("mask", [0, 1, 2])
def test_group_forward_shares_one_prologue(T, mask):
    """q, k and v of one input through tasq_linear_forward_group: each output equals the oracle
    linear of its own layer at its own bit width (8, 5 and 3 here, so members mix the stored and
    the masked-ahead weights)."""
    rng = np.random.default_rng(31)
    n, K, M = 64, 1280, 700
    shapes = [1280, 640, 2000]
    layers = []
    for N in shapes:
        w = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
        s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
        layers.append((N, K, w, s_w))
    layers.append((512, 640, rng.integers(-127, 128, size=(512, 640)).astype(np.int8), np.ones(512, np.float32)))
    ctx = _ctx(T, layers, 2, n, M)
    T.tasq_debug_set_mask_mode(ctx, mask)
    sched = np.array([[8, 8], [5, 8], [3, 8], [8, 8]], np.uint8)
    T.tasq_set_schedule(ctx, sched, _stream())
    x = _acts(rng, M, K)
    xd = _dev(x)
    ldys = [N + 8 for N in shapes]
    ys = [torch.full((M, ld), float("nan"), dtype=torch.float16, device="cuda") for ld in ldys]
    T.tasq_linear_forward_group(ctx, xd, M, K, [0, 1, 2], 0, ys, ldys, _stream())
    torch.cuda.synchronize()
    for (N, _, w, s_w), y, bits in zip(layers, ys, (8, 5, 3)):
        got_all = y.float().cpu().numpy()
        assert np.isnan(got_all[:, N:]).all(), "write past column N"
        got = got_all[:, :N].astype(np.float64)
        ref = oracle.masked_linear(x, w, s_w, bits, n)["y"]
        assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY), f"layer with bits={bits}"
    assert T.tasq_get_device_status(ctx) == 0

    def err(*a):
        with pytest.raises(T.TasqError) as ei:
            T.tasq_linear_forward_group(ctx, *a)
        return ei.value.status

    y0 = ys[0]
    assert err(xd, M, K, [0, 3], 0, [y0, y0], [ldys[0], ldys[0]], _stream()) == T.TASQ_ERR_INVALID_ARG  # K differs
    assert err(xd, M, K, [0, 1, 2, 0, 1], 0, [y0] * 5, [2008] * 5, _stream()) == T.TASQ_ERR_INVALID_ARG  # > 4
    assert err(xd, M, K, [0, 1], 2, [y0, y0], [ldys[0], 2008], _stream()) == T.TASQ_ERR_INVALID_ARG      # step


def test_forward_replays_from_a_cuda_graph(T):
    """Forwards captured in a CUDA graph (prologue with the weight pass, then the GEMM, linked by
    programmatic launch) replay to the same bits as the same forwards launched directly."""
    rng = np.random.default_rng(41)
    n, K, N, M = 64, 1152, 1152, 512
    x = _acts(rng, M, K)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    ctx = _ctx(T, [(N, K, w, s_w), (N, K, w[::-1].copy(), s_w)], 2, n, M)
    T.tasq_set_schedule(ctx, np.array([[5, 8], [8, 3]], np.uint8), _stream())
    xd = _dev(x)
    eager = [torch.empty((M, N), dtype=torch.float16, device="cuda") for _ in range(2)]
    for layer in range(2):
        T.tasq_linear_forward(ctx, xd, M, K, layer, layer, eager[layer], N, _stream())
    torch.cuda.synchronize()
    replay = [torch.zeros((M, N), dtype=torch.float16, device="cuda") for _ in range(2)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for layer in range(2):
            T.tasq_linear_forward(ctx, xd, M, K, layer, layer, replay[layer], N, torch.cuda.current_stream())
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager, replay):
        assert torch.equal(a, b)
    ref = oracle.masked_linear(x, w, s_w, 5, n)["y"]
    got = replay[0].float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY)
    assert T.tasq_get_device_status(ctx) == 0


def test_back_to_back_forwards_with_changing_token_counts(T):
    """Back-to-back forwards on one stream whose token count changes every call, with and without
    the weight pass, no synchronisation until the end: each forward reuses the workspace and the
    masked-weight buffer after the one before it."""
    rng = np.random.default_rng(55)
    n, K, N = 64, 1152, 640
    w = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    Ms = [1000, 37, 1500, 256, 1, 999, 1500]
    ctx = _ctx(T, [(N, K, w, s_w)], 2, n, max(Ms))
    T.tasq_set_schedule(ctx, np.array([[8, 4]], np.uint8), _stream())
    jobs = []
    for i, M in enumerate(Ms):
        x = _acts(rng, M, K)
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        T.tasq_linear_forward(ctx, _dev(x), M, K, 0, i % 2, y, N, _stream())
        jobs.append((x, y, 8 if i % 2 == 0 else 4))
    torch.cuda.synchronize()
    for x, y, bits in jobs:
        ref = oracle.masked_linear(x, w, s_w, bits, n)["y"]
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY), (x.shape[0], bits)
    assert T.tasq_get_device_status(ctx) == 0


def test_schedule_is_stream_ordered(T):
    """A schedule change between two forwards on one stream affects only the later forward, and
    the weights are never rewritten (the same buffer serves both)."""
    rng = np.random.default_rng(3)
    M, K, N, n = 256, 1152, 1152, 64
    x = _acts(rng, M, K)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    ctx = _ctx(T, [(N, K, w, s_w)], 1, n, M)
    xd = _dev(x)
    ys = [torch.empty((M, N), dtype=torch.float16, device="cuda") for _ in range(3)]
    s = _stream()
    T.tasq_set_schedule(ctx, np.array([[8]], np.uint8), s)
    T.tasq_linear_forward(ctx, xd, M, K, 0, 0, ys[0], N, s)
    T.tasq_set_schedule(ctx, np.array([[3]], np.uint8), s)
    T.tasq_linear_forward(ctx, xd, M, K, 0, 0, ys[1], N, s)
    T.tasq_set_schedule(ctx, np.array([[8]], np.uint8), s)
    T.tasq_linear_forward(ctx, xd, M, K, 0, 0, ys[2], N, s)
    torch.cuda.synchronize()
    for y, bits in zip(ys, (8, 3, 8)):
        ref = oracle.masked_linear(x, w, s_w, bits, n)["y"]
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY)
    assert torch.equal(ys[0], ys[2])


@pytest.mark.parametrize("mask", [0, 1, 2])
def test_multi_layer_context_uses_each_layers_weights(T, mask):
    """Every (layer, step) of a 4 x 3 schedule enqueued back to back on one stream before a single
    synchronize: forwards of different layers reuse the context's workspace and masked-weight
    buffer, so each kernel must wait for the one before it that reads them."""
    rng = np.random.default_rng(9)
    n, M = 64, 200
    shapes = [(1152, 3456), (1152, 1152), (4608, 1152), (64, 200)]
    layers, xs = [], []
    for K, N in shapes:
        w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
        s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
        layers.append((N, K, w, s_w))
        xs.append(_acts(rng, M, K))
    ctx = _ctx(T, layers, 3, n, M)
    T.tasq_debug_set_mask_mode(ctx, mask)
    sched = np.array([[8, 4, 6], [5, 8, 2], [7, 7, 1], [1, 2, 3]], np.uint8)
    T.tasq_set_schedule(ctx, sched, _stream())
    xds = [_dev(x) for x in xs]
    outs = {}
    for step in range(3):
        for layer, (N, K, _, _) in enumerate(layers):
            assert T.tasq_layer_info(ctx, layer) == (N, K, K)
            y = torch.empty((M, N), dtype=torch.float16, device="cuda")
            T.tasq_linear_forward(ctx, xds[layer], M, K, layer, step, y, N, _stream())
            outs[layer, step] = y
    torch.cuda.synchronize()
    for (layer, step), y in outs.items():
        N, K, w, s_w = layers[layer]
        ref = oracle.masked_linear(xs[layer], w, s_w, int(sched[layer, step]), n)["y"]
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY), (layer, step)
    assert T.tasq_get_device_status(ctx) == 0


def test_bf16_forward(T):
    rng = np.random.default_rng(21)
    M, K, N, n = 130, 2240, 700, 128
    Kp = oracle.padded_k(K, n)
    x = _acts(rng, M, K)
    w = rng.integers(-127, 128, size=(N, Kp)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    ctx = _ctx(T, [(N, K, w, s_w)], 1, n, M, out=1)
    T.tasq_set_schedule(ctx, np.array([[6]], np.uint8), _stream())
    ldy = 704                       # N = 700 is ragged; the row stride must be a multiple of 8
    y = torch.empty((M, ldy), dtype=torch.bfloat16, device="cuda")
    T.tasq_linear_forward(ctx, _dev(x), M, K, 0, 0, y, ldy, _stream())
    torch.cuda.synchronize()
    ref = oracle.masked_linear(x, w, s_w, 6, n)["y"]
    got = y[:, :N].float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + ABS_TINY)


# ----------------------------------------------------------------------------- errors and status
def test_argument_errors_on_device(T):
    rng = np.random.default_rng(1)
    M, K, N = 64, 128, 64
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    ctx = _ctx(T, [(N, K, w, np.ones(N, np.float32))], 2, 64, M)
    x = torch.zeros((M + 1, K), dtype=torch.float16, device="cuda")
    y = torch.zeros((M + 1, N + 8), dtype=torch.float16, device="cuda")
    s = _stream()

    def err(fn, *a):
        with pytest.raises(T.TasqError) as ei:
            fn(*a)
        return ei.value.status

    assert err(T.tasq_linear_forward, ctx, x, M + 1, K, 0, 0, y, N, s) == T.TASQ_ERR_WORKSPACE
    assert err(T.tasq_linear_forward, ctx, x.data_ptr() + 2, M, K, 0, 0, y, N, s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_linear_forward, ctx, x, M, K - 4, 0, 0, y, N, s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_linear_forward, ctx, x, M, K, 1, 0, y, N, s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_linear_forward, ctx, x, M, K, 0, 2, y, N, s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_linear_forward, ctx, x, M, K, 0, -1, y, N, s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_linear_forward, ctx, x, M, K, 0, 0, y, N + 3, s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_linear_forward, ctx, x, -1, K, 0, 0, y, N, s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_set_schedule, ctx, np.array([[8, 10]], np.uint8), s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_set_schedule, ctx, np.array([[9, 8]], np.uint8), s) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_debug_set_gemm_mode, ctx, 3) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_debug_set_mask_mode, ctx, 3) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_debug_set_mask_mode, ctx, -1) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_debug_set_prologue_mode, ctx, 4) == T.TASQ_ERR_INVALID_ARG
    T.tasq_linear_forward(ctx, x, 0, K, 0, 0, y, N, s)        # M = 0: nothing to do
    assert T.tasq_get_device_status(ctx) == 0
    with pytest.raises(T.TasqError):
        T.tasq_linear_create([(N, 12, w, np.ones(N, np.float32))], 1, 64, 8)   # K % 8 != 0
    with pytest.raises(T.TasqError):
        T.tasq_linear_create([(N, 16392, np.zeros((N, 16448), np.int8), np.ones(N, np.float32))], 1, 64, 8)


def test_stuck_wait_times_out_and_context_stays_usable(T):
    """A wait on a barrier nothing arrives on runs out, reports a status bit, and the context
    keeps working afterwards (failure detected on the host, no fault, no trap)."""
    rng = np.random.default_rng(5)
    M, K, N, n = 256, 1152, 256, 64
    x = _acts(rng, M, K)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    ctx = _ctx(T, [(N, K, w, s_w)], 1, n, M)
    T.tasq_set_wait_limit(ctx, 20_000_000)       # 20 ms
    T.tasq_debug_stuck_wait(ctx, _stream())
    st = T.tasq_get_device_status(ctx, clear=True)
    assert st & T.TASQ_DEVICE_TIMEOUT_MMA
    assert T.tasq_get_device_status(ctx) == 0
    T.tasq_set_wait_limit(ctx, 1_000_000_000)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    T.tasq_linear_forward(ctx, _dev(x), M, K, 0, 0, y, N, _stream())
    torch.cuda.synchronize()
    ref = oracle.masked_linear(x, w, s_w, 8, n)["y"]
    assert np.all(np.abs(y.float().cpu().numpy() - ref) <= F16_REL * np.abs(ref) + ABS_TINY)
    assert T.tasq_get_device_status(ctx) == 0


def test_trace_counts_launches(T):
    rng = np.random.default_rng(8)
    M, K, N = 256, 1152, 1152
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    ctx = _ctx(T, [(N, K, w, np.ones(N, np.float32))], 1, 64, M)
    T.tasq_trace_enable(ctx, 4)
    x = _dev(_acts(rng, M, K))
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    for _ in range(6):
        T.tasq_linear_forward(ctx, x, M, K, 0, 0, y, N, _stream())
    tr = T.tasq_trace_read(ctx)
    assert tr["gemm_launches"] == 4 and tr["prologue_launches"] == 4
    assert tr["gemm_ms"] > 0 and tr["prologue_ms"] > 0
    assert tr["gemm_ops"] == 4 * 2.0 * M * N * K


def test_two_host_threads_two_contexts(T):
    """Two host threads, each with its own context and stream, run INT8 and NVFP4 forwards at the
    same time (run alone, both threads also reach the launchers' one-time per-device set-up of
    shared-memory limits and resident CTA pairs together). Every output equals the oracle's: the
    set-up is guarded, and contexts share no device state."""
    import threading
    n, M = 64, 700
    shapes = [(1152, 4608), (4608, 1152)]        # the CTA-pair and the one-CTA INT8 GEMM
    rng = np.random.default_rng(404)
    jobs = []
    for K, N in shapes:
        w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
        s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
        jobs.append((K, N, w, s_w, _acts(rng, M, K)))
    bits = [8, 5, 0, 3]                             # INT8 widths and an NVFP4 step
    outs = [None, None]
    errors = []

    def run(i):
        try:
            K, N, w, s_w, x = jobs[i]
            stream = torch.cuda.Stream()
            ctx = T.tasq_linear_create([(N, K, w, s_w)], len(bits), n, M, 0, stream)
            T.tasq_debug_set_gemm_mode(ctx, 2 if i == 0 else 1)
            T.tasq_set_schedule(ctx, np.array([bits], np.uint8), stream)
            xd = torch.from_numpy(x).cuda()
            ys = []
            for step in range(len(bits)):
                y = torch.empty((M, N), dtype=torch.float16, device="cuda")
                T.tasq_linear_forward(ctx, xd, M, K, 0, step, y, N, stream)
                ys.append(y)
            stream.synchronize()
            outs[i] = ([y.float().cpu().numpy().astype(np.float64) for y in ys], T.tasq_get_device_status(ctx))
            T.tasq_linear_destroy(ctx)
        except Exception as e:   # reported on the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    for i, (K, N, w, s_w, x) in enumerate(jobs):
        ys, status = outs[i]
        assert status == 0
        for step, b in enumerate(bits):
            if b == 0:
                r4 = oracle.nvfp4_linear(x, w, s_w, n)
                tol = (K * 2.0 ** -24 * oracle.nvfp4_abs_terms(r4["ca"], r4["sa"], r4["cw"], r4["sw"]) * 1.0001 *
                       r4["s_x"][:, None] * s_w[None, :] + np.abs(r4["y"]) * (2.0 ** -11 + 2.0 ** -21) + ABS_TINY)
                assert np.all(np.abs(ys[step] - r4["y"]) <= tol), f"thread {i} NVFP4 step"
            else:
                ref = oracle.masked_linear(x, w, s_w, b, n)["y"]
                assert np.linalg.norm(ys[step] - ref) <= 1e-3 * np.linalg.norm(ref), f"thread {i} bits {b}"
