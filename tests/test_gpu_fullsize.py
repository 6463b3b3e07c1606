"""Full-size parity: every distinct layer shape of every workload at its full token count, run
through tasq_linear_forward exactly as the bench launches it, checked on a seeded sample of
token rows (plus the whole last, ragged token tile) against the oracle computed row by row.
Each layer runs at every bit width its schedule gives it (a (layer, step) result depends on the
step only through that width), and the NVFP4 workload's layers also in their NVFP4 step."""
import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from conftest import build_library
    t = build_library()
    return t


@pytest.mark.parametrize("name", workloads.WORKLOAD_ORDER)
def test_fullsize_workload(T, name):
    wl = workloads.WORKLOADS[name]
    M, n = wl.tokens, wl.hadamard_n
    sched = workloads.schedule(wl)
    # one context layer per distinct (K, N) of the block, in block order
    picked, seen = [], set()
    for j, (lname, K, N) in enumerate(wl.block_layers):
        if (K, N) not in seen:
            seen.add((K, N))
            picked.append(j)
    layers, xs = [], []
    for j in picked:
        _, K, N = wl.layer_shape(j)
        w, s_w = workloads.weights(wl, j)
        layers.append((N, K, w, s_w))
        xs.append(workloads.activations(wl, j))
    # step t of the test table runs width 8 - t: every width a layer's schedule uses is one step
    widths = [sorted({int(v) for v in sched[j::len(wl.block_layers)].ravel()}, reverse=True) for j in picked]
    table = np.array([[8 - t for t in range(8)] for _ in picked], np.uint8)
    s = torch.cuda.current_stream()
    ctx = T.tasq_linear_create(layers, 8, n, M, 0, s)
    T.tasq_set_schedule(ctx, table, s)
    rows = workloads.sample_rows(M)
    for li, ((N, K, w, s_w), x) in enumerate(zip(layers, xs)):
        Kp = oracle.padded_k(K, n)
        xd = torch.from_numpy(x).cuda()
        # codes of the sampled rows
        xq = torch.empty((M, Kp), dtype=torch.int8, device="cuda")
        sx = torch.empty((M,), dtype=torch.float32, device="cuda")
        T.tasq_debug_quantize(ctx, xd, M, K, li, xq, sx, s)
        torch.cuda.synchronize()
        q_ref, sx_ref, _ = oracle.prologue(x[rows], n)
        q_got = xq.cpu().numpy()[rows]
        d = np.abs(q_got.astype(np.int64) - q_ref.astype(np.int64))
        assert d.max() <= 1 and d.astype(bool).mean() <= 1e-3
        assert np.all(np.abs(sx.cpu().numpy()[rows] - sx_ref) <= 1e-6 * np.abs(sx_ref))
        del xq
        for bits in widths[li]:
            step = 8 - bits
            y = torch.empty((M, N), dtype=torch.float16, device="cuda")
            T.tasq_linear_forward(ctx, xd, M, K, li, step, y, N, s)
            torch.cuda.synchronize()
            got = y[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
            ref = oracle.dequant(oracle.int_gemm(q_ref, oracle.lsb_mask(w, bits)), sx_ref, s_w)
            assert np.linalg.norm(got - ref) <= 1e-3 * np.linalg.norm(ref), (name, li, bits)
            exact_rows = ~(d.any(axis=1))
            assert np.all(np.abs(got[exact_rows] - ref[exact_rows]) <= 1e-3 * np.abs(ref[exact_rows]) + 2.0 ** -24)
            assert np.all(np.isfinite(y.float().cpu().numpy())), "non-finite output"
            del y
        del xd
    assert T.tasq_get_device_status(ctx) == 0
    T.tasq_linear_destroy(ctx)


def test_fullsize_nvfp4_workload(T):
    """CogVideoX with its stable blocks in NVFP4: every distinct layer shape at the full 17776
    tokens in its NVFP4 step, on sampled rows, within the FP32 accumulation bound."""
    wl = workloads.WORKLOADS["cogvideox_nvfp4"]
    M, n = wl.tokens, wl.hadamard_n
    assert (workloads.schedule(wl) == 0).any()
    rows = workloads.sample_rows(M)
    s = torch.cuda.current_stream()
    seen = set()
    for j, (lname, K, N) in enumerate(wl.block_layers):
        if (K, N) in seen:
            continue
        seen.add((K, N))
        w, s_w = workloads.weights(wl, j)
        x = workloads.activations(wl, j)
        ctx = T.tasq_linear_create([(N, K, w, s_w)], 1, n, M, 0, s)
        T.tasq_set_schedule(ctx, np.array([[0]], np.uint8), s)
        xd = torch.from_numpy(x).cuda()
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        T.tasq_linear_forward(ctx, xd, M, K, 0, 0, y, N, s)
        torch.cuda.synchronize()
        got = y[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
        r = oracle.nvfp4_linear(x[rows], w, s_w, n)
        Kp = oracle.padded_k(K, n)
        bound = (Kp * 2.0 ** -24 * oracle.nvfp4_abs_terms(r["ca"], r["sa"], r["cw"], r["sw"]) * 1.0001 *
                 r["s_x"][:, None] * s_w[None, :] + np.abs(r["y"]) * (2.0 ** -11 + 2.0 ** -21) + 2.0 ** -24)
        assert np.all(np.abs(got - r["y"]) <= bound), lname
        assert np.all(np.isfinite(y.float().cpu().numpy())), "non-finite output"
        assert T.tasq_get_device_status(ctx) == 0
        T.tasq_linear_destroy(ctx)
        del xd, y


# (GEMM kernel, mask placement) pairs of the full-size INT32 check: kernel 1 = one CTA per
# 128 x 256 tile, 2 = CTA pairs on 256 x 256 tiles; placement 1 = inside the GEMM, 2 = once ahead
FULLSIZE_S32_MODES = [(1, 1), (1, 2), (2, 1), (2, 2)]


@pytest.mark.parametrize("name", [w for w in workloads.WORKLOAD_ORDER if w != "single"])
def test_fullsize_int32_accumulators_bit_exact(T, name):
    """The raw INT32 accumulators of every distinct layer shape of a workload, at its full token
    count and at every bit width its schedule uses, on both GEMM kernels and both mask placements,
    equal the exact integer products of the GPU's own activation codes with the masked weights
    (HQ-DM's integer core, section 2.1 "Eficiencia de Hardware"; TASQ's LSB mask, section 2).
    These launches have many more tiles than CTAs, so every CTA walks several tiles through both
    TMEM accumulators and both accumulator phases. Checked on the sampled rows (the whole last,
    ragged token tile included) and every output channel."""
    wl = workloads.WORKLOADS[name]
    M, n = wl.tokens, wl.hadamard_n
    sched = workloads.schedule(wl)
    per = len(wl.block_layers)
    picked, seen = [], set()
    for j, (lname, K, N) in enumerate(wl.block_layers):
        if (K, N) not in seen:
            seen.add((K, N))
            picked.append(j)
    rows = workloads.sample_rows(M)
    rows_d = torch.from_numpy(rows).cuda()
    s = torch.cuda.current_stream()
    for j in picked:
        _, K, N = wl.layer_shape(j)
        w, s_w = workloads.weights(wl, j)
        x = workloads.activations(wl, j)
        Kp = oracle.padded_k(K, n)
        widths = sorted({int(v) for v in sched[j::per].ravel()} - {0}, reverse=True)
        ctx = T.tasq_linear_create([(N, K, w, s_w)], 8, n, M, 0, s)
        T.tasq_set_schedule(ctx, np.array([[8 - t for t in range(8)]], np.uint8), s)
        xq = torch.empty((M, Kp), dtype=torch.int8, device="cuda")
        sx = torch.empty((M,), dtype=torch.float32, device="cuda")
        T.tasq_debug_quantize(ctx, torch.from_numpy(x).cuda(), M, K, 0, xq, sx, s)
        torch.cuda.synchronize()
        q_rows = xq[rows_d].cpu().numpy()
        ld = N + (8 - N % 8) % 8
        acc = torch.empty((M, ld), dtype=torch.int32, device="cuda")
        for bits in widths:
            ref = oracle.int_gemm(q_rows, oracle.lsb_mask(w, bits))
            for gemm, mask in FULLSIZE_S32_MODES:
                T.tasq_debug_set_gemm_mode(ctx, gemm)
                T.tasq_debug_set_mask_mode(ctx, mask)
                acc.fill_(0x7F7F7F7F)
                T.tasq_debug_gemm_s32(ctx, xq, M, 0, 8 - bits, acc, ld, s)
                torch.cuda.synchronize()
                got = acc[rows_d, :N].cpu().numpy().astype(np.int64)
                bad = np.argwhere(got != ref)
                assert bad.size == 0, (name, K, N, bits, gemm, mask, bad[:4].tolist())
        assert T.tasq_get_device_status(ctx) == 0
        T.tasq_linear_destroy(ctx)
        del xq, acc
