"""NVFP4 steps on the GPU against the oracle (6Bit-Diffusion's stable layers in NVFP4).

The prologue and the weight conversion take every floating-point decision in FP32 in the
oracle's order, so codes and block scales must agree bit for bit. The block-scaled GEMM
accumulates in FP32 in the tensor core's own order: its accumulators must lie within
Kp * 2^-24 * sum |terms| of the exact sum, and y within that bound carried through the scales
plus the FP16 rounding of the output."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def T():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from conftest import build_library
    return build_library()


def _stream():
    return torch.cuda.current_stream()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _acts(rng, M, K):
    x = rng.standard_normal((M, K)).astype(np.float32)
    cols = rng.choice(K, size=max(1, K // 200), replace=False)
    x[:, cols] *= 50.0
    return x.astype(np.float16)


def _kp4(Kp):
    return -(-Kp // 256) * 256


def unchunk_scales(buf, rows, Kp):
    """[rows, Kp/16] scale bytes out of the chunked layout of include/tasq.h (layout only)."""
    chunks = _kp4(Kp) // 64
    b = np.asarray(buf, dtype=np.uint8).reshape(-1, chunks, 512)
    r = np.arange(rows)[:, None]
    j = np.arange(Kp // 16)[None, :]
    return b[r // 128, j // 4, (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)]


def chunk_scales(sf, Kp):
    """The inverse: [rows, Kp/16] scale bytes into the chunked layout, zero elsewhere."""
    rows = sf.shape[0]
    chunks = _kp4(Kp) // 64
    groups = -(-rows // 128)
    b = np.zeros((groups, chunks, 512), np.uint8)
    r = np.arange(rows)[:, None]
    j = np.arange(Kp // 16)[None, :]
    b[r // 128, j // 4, (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)] = sf
    return b.reshape(-1)


def _ctx(T, layers, steps, n, max_tokens):
    return T.tasq_linear_create(layers, steps, n, max_tokens, 0, _stream())


# ----------------------------------------------------------------------------- prologue
@pytest.mark.parametrize("n,K,M", [(64, 64, 1), (64, 1152, 257), (128, 2240, 130), (64, 4608, 300),
                                   (64, 12288, 33), (128, 10240, 40), (128, 5600, 64), (64, 1280, 4097),
                                   (64, 96, 3)])
def test_nvfp4_prologue_matches_oracle(T, n, K, M):
    rng = np.random.default_rng(K + 7 * M)
    x = _acts(rng, M, K)
    if M >= 3:
        x[1] = 0
        x[2, ::5] = np.float16(2.0 ** -20)    # FP16 subnormals
    Kp = oracle.padded_k(K, n)
    ctx = _ctx(T, [(64, K, np.zeros((64, Kp), np.int8), np.ones(64, np.float32))], 1, n, M)
    codes = torch.empty((M, Kp // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((T.tasq_nvfp4_scale_bytes(M, Kp),), dtype=torch.uint8, device="cuda")
    sx = torch.empty((M,), dtype=torch.float32, device="cuda")
    T.tasq_debug_quantize_nvfp4(ctx, _dev(x), M, K, 0, codes, sf, sx, _stream())
    torch.cuda.synchronize()
    c_ref, sb_ref, sx_ref, _ = oracle.nvfp4_prologue(x, n)
    got = oracle.unpack_nibbles(codes.cpu().numpy())
    assert np.array_equal(unchunk_scales(sf.cpu().numpy(), M, Kp), sb_ref), "block scales"
    bad = np.argwhere(got != c_ref)
    assert len(bad) == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}"
    sx_g = sx.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(sx_g - sx_ref) <= 1e-6 * np.abs(sx_ref)), "s_x"
    assert T.tasq_get_device_status(ctx) == 0


def test_nvfp4_prologue_exact_ties(T):
    """Scaled values on exact E2M1 midpoints. Per row, the first Hadamard block of z holds 42 once
    (a = 42, so g = fp32(2688 / 42) = 64 exactly) and the second holds, in each 16-block, small
    multiples of 1/64 whose largest is 0.375: u = 64 z has block maximum 24, so the block scale is
    4 (exact reciprocal) and u / 4 = 16 z are exact halves. x = z H_64 / 64 is exact in FP16 and
    every butterfly of it is exact in FP32."""
    rng = np.random.default_rng(5)
    M, n = 40, 64
    K = 2 * n
    z = np.zeros((M, K))
    z[:, 0] = 42.0
    half = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
    for b in range(4, 8):
        t = rng.choice(half, size=(M, 16)) * rng.choice([-1.0, 1.0], size=(M, 16))
        t[:, 0] = 6.0
        z[:, 16 * b:16 * b + 16] = t / 16.0
    H = oracle.sylvester_hadamard(n).astype(np.float64)
    x = np.concatenate([z[:, b * n:(b + 1) * n] @ H / n for b in range(2)], axis=1)
    assert np.array_equal(x.astype(np.float16).astype(np.float64), x)
    x = x.astype(np.float16)
    ctx = _ctx(T, [(64, K, np.zeros((64, K), np.int8), np.ones(64, np.float32))], 1, n, M)
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((T.tasq_nvfp4_scale_bytes(M, K),), dtype=torch.uint8, device="cuda")
    sx = torch.empty((M,), dtype=torch.float32, device="cuda")
    T.tasq_debug_quantize_nvfp4(ctx, _dev(x), M, K, 0, codes, sf, sx, _stream())
    torch.cuda.synchronize()
    c_ref, sb_ref, _, z32 = oracle.nvfp4_prologue(x, n)
    assert np.array_equal(z32, z.astype(np.float32)), "the transform is exact here"
    assert np.all(sb_ref[:, 4:] == 0x48), "scale 4 in the tie blocks"
    assert np.array_equal(c_ref[:, 64:], oracle.e2m1_encode(16.0 * z[:, 64:])), "oracle: ties to even"
    assert np.array_equal(oracle.unpack_nibbles(codes.cpu().numpy()), c_ref), "ties to even on the GPU"
    assert np.array_equal(unchunk_scales(sf.cpu().numpy(), M, K), sb_ref)


# ----------------------------------------------------------------------------- weights
@pytest.mark.parametrize("N,K,n", [(1, 64, 64), (200, 1152, 64), (130, 2240, 128), (1152, 4608, 64)])
def test_nvfp4_weights_match_oracle(T, N, K, n):
    rng = np.random.default_rng(N + K)
    Kp = oracle.padded_k(K, n)
    w = rng.integers(-128, 128, size=(N, Kp)).astype(np.int8)
    w[0, :16] = 0                              # an all-zero block: scale 0, codes 0
    ctx = _ctx(T, [(N, K, w, np.ones(N, np.float32))], 1, n, 16)
    codes = torch.full((N, Kp // 2), 0xAB, dtype=torch.uint8, device="cuda")
    nbytes = T.tasq_nvfp4_scale_bytes(N, Kp)
    sf = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
    T.tasq_debug_nvfp4_weights(ctx, 0, codes, sf, _stream())
    torch.cuda.synchronize()
    c_ref, sb_ref = oracle.nvfp4_quantize_weights(w)
    assert np.array_equal(oracle.unpack_nibbles(codes.cpu().numpy()), c_ref), "weight codes"
    sfh = sf.cpu().numpy()
    assert np.array_equal(unchunk_scales(sfh, N, Kp), sb_ref), "weight block scales"
    # K padding up to a multiple of 256 holds zero scales
    if _kp4(Kp) > Kp:
        pad = unchunk_scales(sfh, N, _kp4(Kp))[:, Kp // 16:]
        assert not pad.any(), "scales past Kp must be zero"


# ----------------------------------------------------------------------------- GEMM
def _terms_bound(ca, sa, cw, sw, Kp):
    return Kp * 2.0 ** -24 * oracle.nvfp4_abs_terms(ca, sa, cw, sw) + 1e-30


@pytest.mark.parametrize("M,N,K,n", [(1, 8, 64, 64), (130, 200, 1152, 64), (300, 520, 320, 64),
                                     (257, 1152, 4608, 64), (64, 2000, 2240, 128), (513, 384, 12288, 64)])
@pytest.mark.parametrize("mode", [1, 2], ids=["one_cta", "cta_pair"])
def test_nvfp4_gemm_accumulators(T, M, N, K, n, mode):
    rng = np.random.default_rng(M * 3 + N + K)
    Kp = oracle.padded_k(K, n)
    w = rng.integers(-127, 128, size=(N, Kp)).astype(np.int8)
    x = _acts(rng, M, K)
    ca, sa, sx, _ = oracle.nvfp4_prologue(x, n)
    cw, sw = oracle.nvfp4_quantize_weights(w)
    ctx = _ctx(T, [(N, K, w, np.ones(N, np.float32))], 1, n, M)
    T.tasq_debug_set_gemm_mode(ctx, mode)
    codes = _dev(oracle.pack_nibbles(ca))
    sf = _dev(chunk_scales(sa, Kp))
    sxd = _dev(sx.astype(np.float32))
    ld = N + (4 - N % 4) % 4
    acc = torch.full((M, ld), float("nan"), dtype=torch.float32, device="cuda")
    T.tasq_debug_gemm_nvfp4(ctx, codes, sf, sxd, M, 0, acc, ld, T.TASQ_NVFP4_RAW_ACC, _stream())
    torch.cuda.synchronize()
    got = acc.cpu().numpy()[:, :N].astype(np.float64)
    ref = oracle.nvfp4_gemm(ca, sa, cw, sw)
    bound = _terms_bound(ca, sa, cw, sw, Kp)
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"max excess {(err - bound).max()} at {np.unravel_index(np.argmax(err - bound), err.shape)}"
    assert T.tasq_get_device_status(ctx) == 0


# ----------------------------------------------------------------------------- whole forward
@pytest.mark.parametrize("n,K,N,M", [(64, 1152, 1152, 256), (64, 1152, 3456, 300), (128, 2240, 6720, 130),
                                     (64, 4608, 1152, 77), (64, 64, 8, 1)])
@pytest.mark.parametrize("mode", [0, 1, 2], ids=["auto", "one_cta", "cta_pair"])
def test_nvfp4_forward_matches_oracle(T, n, K, N, M, mode):
    rng = np.random.default_rng(n + K + N + M)
    Kp = oracle.padded_k(K, n)
    x = _acts(rng, M, K)
    w = rng.integers(-127, 128, size=(N, Kp)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    bits = [8, T.TASQ_NVFP4, 5, T.TASQ_NVFP4]
    ctx = _ctx(T, [(N, K, w, s_w)], len(bits), n, M + 3)
    T.tasq_debug_set_gemm_mode(ctx, mode)
    T.tasq_set_schedule(ctx, np.array([bits], np.uint8), _stream())
    xd = _dev(x)
    ldy = N + (8 - N % 8) % 8 + 8
    r4 = oracle.nvfp4_linear(x, w, s_w, n)
    bound = _terms_bound(r4["ca"], r4["sa"], r4["cw"], r4["sw"], Kp) * r4["s_x"][:, None] * s_w[None, :]
    for step, b in enumerate(bits):
        y = torch.full((M + 1, ldy), float("nan"), dtype=torch.float16, device="cuda")
        T.tasq_linear_forward(ctx, xd, M, K, 0, step, y, ldy, _stream())
        torch.cuda.synchronize()
        got = y.float().cpu().numpy()
        assert np.all(np.isnan(got[M:])) and np.all(np.isnan(got[:M, N:])), "write outside [M, N]"
        got = got[:M, :N].astype(np.float64)
        if b == T.TASQ_NVFP4:
            ref = r4["y"]
            tol = bound * 1.0001 + np.abs(ref) * (2.0 ** -11 + 2.0 ** -21) + 2.0 ** -24
            assert np.all(np.abs(got - ref) <= tol), f"NVFP4 step {step}"
        else:
            ref = oracle.masked_linear(x, w, s_w, b, n)["y"]
            rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
            assert rel <= 1e-3, f"INT8 step {step}: {rel}"
    assert T.tasq_get_device_status(ctx) == 0


@pytest.mark.parametrize("mode", [1, 2], ids=["one_cta", "cta_pair"])
def test_nvfp4_forward_bf16_output(T, mode):
    """BF16 outputs of an NVFP4 step: the FP32 bound of the accumulators carried through the
    scales, plus the BF16 rounding (8 significant bits: half an ulp is at most 2^-8 of |y|)."""
    rng = np.random.default_rng(77 + mode)
    n, K, N, M = 64, 1152, 1000, 389     # odd and even 192-token tiles, a ragged channel tile
    Kp = oracle.padded_k(K, n)
    x = _acts(rng, M, K)
    w = rng.integers(-127, 128, size=(N, Kp)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    ctx = T.tasq_linear_create([(N, K, w, s_w)], 1, n, M, T.TASQ_OUT_BF16, _stream())
    T.tasq_debug_set_gemm_mode(ctx, mode)
    T.tasq_set_schedule(ctx, np.array([[T.TASQ_NVFP4]], np.uint8), _stream())
    ldy = 1008
    y = torch.full((M + 1, ldy), float("nan"), dtype=torch.bfloat16, device="cuda")
    T.tasq_linear_forward(ctx, _dev(x), M, K, 0, 0, y, ldy, _stream())
    torch.cuda.synchronize()
    got = y.float().cpu().numpy()
    assert np.all(np.isnan(got[M:])) and np.all(np.isnan(got[:M, N:])), "write outside [M, N]"
    got = got[:M, :N].astype(np.float64)
    r4 = oracle.nvfp4_linear(x, w, s_w, n)
    bound = _terms_bound(r4["ca"], r4["sa"], r4["cw"], r4["sw"], Kp) * r4["s_x"][:, None] * s_w[None, :]
    tol = bound * 1.0001 + np.abs(r4["y"]) * (2.0 ** -8 + 2.0 ** -21) + 2.0 ** -24
    assert np.all(np.abs(got - r4["y"]) <= tol)
    assert T.tasq_get_device_status(ctx) == 0


def test_nvfp4_and_int8_layers_interleave(T):
    """Two layers, NVFP4 and INT8 steps back to back on one stream: each forward reads its own
    weights, the NVFP4 weights never leak into the INT8 path (they share the masked-weight slot)."""
    rng = np.random.default_rng(31)
    n, M = 64, 200
    shapes = [(1152, 768), (768, 1152)]
    layers, ws = [], []
    for K, N in shapes:
        w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
        s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
        layers.append((N, K, w, s_w))
        ws.append((w, s_w))
    ctx = _ctx(T, layers, 3, n, M)
    sched = np.array([[0, 4, 0], [8, 0, 3]], np.uint8)
    T.tasq_set_schedule(ctx, sched, _stream())
    xs = [_acts(rng, M, K) for K, _ in shapes]
    outs = []
    for step in range(3):
        for l in range(2):
            K, N = shapes[l]
            y = torch.empty((M, N), dtype=torch.float16, device="cuda")
            T.tasq_linear_forward(ctx, _dev(xs[l]), M, K, l, step, y, N, _stream())
            outs.append((l, step, y))
    torch.cuda.synchronize()
    for l, step, y in outs:
        w, s_w = ws[l]
        b = int(sched[l, step])
        got = y.float().cpu().numpy().astype(np.float64)
        if b == 0:
            r = oracle.nvfp4_linear(xs[l], w, s_w, n)
            Kp = shapes[l][0]
            tol = (_terms_bound(r["ca"], r["sa"], r["cw"], r["sw"], Kp) * r["s_x"][:, None] * s_w[None, :] * 1.0001 +
                   np.abs(r["y"]) * (2.0 ** -11 + 2.0 ** -21) + 2.0 ** -24)
            assert np.all(np.abs(got - r["y"]) <= tol), f"layer {l} step {step} (NVFP4)"
        else:
            ref = oracle.masked_linear(xs[l], w, s_w, b, n)["y"]
            assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-3, f"layer {l} step {step} (INT8)"
    assert T.tasq_get_device_status(ctx) == 0


def test_nvfp4_argument_errors(T):
    ctx = _ctx(T, [(64, 64, np.zeros((64, 64), np.int8), np.ones(64, np.float32))], 1, 64, 16)
    codes = torch.empty((16, 32), dtype=torch.uint8, device="cuda")
    sf = torch.empty((T.tasq_nvfp4_scale_bytes(16, 64),), dtype=torch.uint8, device="cuda")
    sx = torch.empty((16,), dtype=torch.float32, device="cuda")
    y = torch.empty((16, 64), dtype=torch.float32, device="cuda")

    def err(fn, *a):
        with pytest.raises(T.TasqError) as ei:
            fn(*a)
        return ei.value.status

    assert err(T.tasq_debug_gemm_nvfp4, ctx, codes, sf, sx, 16, 0, y, 64, 7, _stream()) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_debug_gemm_nvfp4, ctx, codes, sf, sx, 16, 0, y, 62, T.TASQ_NVFP4_RAW_ACC, _stream()) == \
        T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_debug_gemm_nvfp4, ctx, codes, sf, sx, 16, 1, y, 64, T.TASQ_NVFP4_RAW_ACC, _stream()) == \
        T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_nvfp4_scale_bytes, 8, 100) == T.TASQ_ERR_INVALID_ARG
    assert err(T.tasq_set_schedule, ctx, np.array([[9]], np.uint8), _stream()) == T.TASQ_ERR_INVALID_ARG


def _nvfp4_tol(r, s_w, Kp):
    return (_terms_bound(r["ca"], r["sa"], r["cw"], r["sw"], Kp) * r["s_x"][:, None] * s_w[None, :] * 1.0001 +
            np.abs(r["y"]) * (2.0 ** -11 + 2.0 ** -21) + 2.0 ** -24)


def test_nvfp4_in_a_group_forward(T):
    """A group whose step is NVFP4 for one member runs every member as its own forward: each
    output equals that member's oracle linear (NVFP4 or INT8)."""
    rng = np.random.default_rng(37)
    n, K, M = 64, 1280, 300
    shapes = [1280, 640, 896]
    layers = []
    for N in shapes:
        w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
        s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
        layers.append((N, K, w, s_w))
    ctx = _ctx(T, layers, 1, n, M)
    T.tasq_set_schedule(ctx, np.array([[8], [0], [5]], np.uint8), _stream())
    x = _acts(rng, M, K)
    ys = [torch.empty((M, N), dtype=torch.float16, device="cuda") for N in shapes]
    T.tasq_linear_forward_group(ctx, _dev(x), M, K, [0, 1, 2], 0, ys, list(shapes), _stream())
    torch.cuda.synchronize()
    for (N, _, w, s_w), y, b in zip(layers, ys, (8, 0, 5)):
        got = y.float().cpu().numpy().astype(np.float64)
        if b == 0:
            r = oracle.nvfp4_linear(x, w, s_w, n)
            assert np.all(np.abs(got - r["y"]) <= _nvfp4_tol(r, s_w, K)), "NVFP4 member"
        else:
            ref = oracle.masked_linear(x, w, s_w, b, n)["y"]
            assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-3, f"INT8 member, bits {b}"
    assert T.tasq_get_device_status(ctx) == 0


def test_nvfp4_forward_replays_from_a_cuda_graph(T):
    """NVFP4 and INT8 forwards captured in one CUDA graph replay to the bits of the direct launches."""
    rng = np.random.default_rng(43)
    n, K, N, M = 64, 1152, 1152, 512
    x = _acts(rng, M, K)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    ctx = _ctx(T, [(N, K, w, s_w)], 2, n, M)
    T.tasq_set_schedule(ctx, np.array([[0, 6]], np.uint8), _stream())
    xd = _dev(x)
    eager = [torch.empty((M, N), dtype=torch.float16, device="cuda") for _ in range(2)]
    for step in range(2):
        T.tasq_linear_forward(ctx, xd, M, K, 0, step, eager[step], N, _stream())
    torch.cuda.synchronize()
    replay = [torch.zeros((M, N), dtype=torch.float16, device="cuda") for _ in range(2)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for step in range(2):
            T.tasq_linear_forward(ctx, xd, M, K, 0, step, replay[step], N, torch.cuda.current_stream())
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager, replay):
        assert torch.equal(a, b)
    assert T.tasq_get_schedule(ctx).reshape(-1).tolist() == [0, 6], "the table keeps the NVFP4 entry"
    assert T.tasq_get_device_status(ctx) == 0
