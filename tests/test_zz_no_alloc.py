"""The allocation-free entry point, tasq_linear_forward_noalloc, against the oracle and against
tasq_linear_forward.

Some callers cannot call cudaMalloc: code running inside an allocator callback, hosts that give
all device memory to their own arena, or harnesses that forbid allocation. They call
tasq_linear_forward_noalloc, which takes the weights directly and keeps the activation codes in
a fixed device array inside the library. This file is collected last on purpose, so that a run
stopping at the first failure has already run every other test. It must pass alone in a fresh
process and after the other tests: the fixed array keeps whatever the previous call left there.
"""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

F16_REL = 1e-3
BF16_REL = 2.0 ** -8
ABS_TINY = 2.0 ** -24
SCRATCH_CONTROL = 256   # control block at the start of the fixed array


@pytest.fixture(scope="module")
def T():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from conftest import build_library
    t = build_library()
    return t


def _case(seed, M, K, N, n):
    rng = np.random.default_rng(seed)
    Kp = -(-K // n) * n
    x = rng.standard_normal((M, K), dtype=np.float32)
    x[:, rng.choice(K, size=max(1, K // 200), replace=False)] *= 50
    w = rng.integers(-128, 128, size=(N, Kp)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    return x.astype(np.float16), w, s_w


def _need(M, Kp):
    """Bytes of the fixed array one call uses: control block and scales rounded up to 1 KiB, then
    the codes."""
    return -(-(SCRATCH_CONTROL + 4 * M) // 1024) * 1024 + M * Kp


def _reference(T, x, w, s_w, N, K, n, bits, ldy):
    """The same layer through the context-based entry point."""
    M = x.shape[0]
    s = torch.cuda.current_stream()
    ctx = T.tasq_linear_create([(N, K, w, s_w)], 1, n, M, T.TASQ_OUT_F16, s)
    T.tasq_set_schedule(ctx, np.array([[bits]], np.uint8), s)
    y = torch.zeros((M, ldy), dtype=torch.float16, device="cuda")
    T.tasq_linear_forward(ctx, torch.from_numpy(x).cuda(), M, K, 0, 0, y, ldy, s)
    torch.cuda.synchronize()
    T.tasq_linear_destroy(ctx)
    return y[:, :N].float().cpu().numpy().astype(np.float64)


def test_noalloc_matches_context_forward_on_two_calls_in_a_row(T):
    s = torch.cuda.current_stream()
    cases = [
        # (seed, M, K, N, n, bits): the second call is smaller in places and larger in others,
        # so it runs over scratch contents the first call left behind
        (11, 300, 1152, 1152, 64, 5),
        (12, 1000, 2240, 704, 128, 3),
    ]
    refs, outs = [], []
    for seed, M, K, N, n, bits in cases:
        x, w, s_w = _case(seed, M, K, N, n)
        refs.append(_reference(T, x, w, s_w, N, K, n, bits, N + 8))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, (seed, M, K, N, n, bits) in enumerate(cases):
        x, w, s_w = _case(seed, M, K, N, n)
        xd = torch.from_numpy(x).cuda()
        wd = torch.from_numpy(w).cuda()
        swd = torch.from_numpy(s_w).cuda()
        y = torch.zeros((M, N + 8), dtype=torch.float16, device="cuda")
        T.tasq_linear_forward_noalloc(xd, M, K, K, wd, swd, N, bits, n, y, N + 8, T.TASQ_OUT_F16,
                                      status if i == 0 else None, s)
        torch.cuda.synchronize()
        outs.append(y[:, :N].float().cpu().numpy().astype(np.float64))
        assert not y[:, N:].any().item(), "write past column N"
    assert int(status.item()) == 0
    for got, ref in zip(outs, refs):
        assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY)


def test_noalloc_matches_the_oracle_at_every_edge_width(T):
    """Calls in a row, each over what the previous one left in the fixed array, checked element by
    element against the oracle's masked linear (TASQ's LSB mask on the caller's weights, HQ-DM's
    block-Hadamard INT8 activations): widths 8, 7, 4 and 1, ragged token counts and channel
    counts (700 and 520 end inside a tile; 700 * 2 bytes is not a whole number of 16-byte output
    granules), FP16 and BF16 outputs, with and without a device status word of the caller's."""
    s = torch.cuda.current_stream()
    cases = [
        # (seed, M, K, N, n, bits, out dtype, caller's status word)
        (21, 300, 1152, 1152, 64, 8, T.TASQ_OUT_F16, True),
        (22, 1000, 2240, 700, 128, 7, T.TASQ_OUT_BF16, False),
        (23, 257, 4608, 520, 64, 4, T.TASQ_OUT_F16, False),
        (24, 77, 640, 1152, 64, 1, T.TASQ_OUT_BF16, True),
    ]
    for seed, M, K, N, n, bits, out, own_status in cases:
        x, w, s_w = _case(seed, M, K, N, n)
        ldy = N + (8 - N % 8) % 8 + 8
        tdt = torch.float16 if out == T.TASQ_OUT_F16 else torch.bfloat16
        y = torch.full((M + 1, ldy), float("nan"), dtype=tdt, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda") if own_status else None
        T.tasq_linear_forward_noalloc(torch.from_numpy(x).cuda(), M, K, K, torch.from_numpy(w).cuda(),
                                      torch.from_numpy(s_w).cuda(), N, bits, n, y, ldy, out, status, s)
        torch.cuda.synchronize()
        got_all = y.float().cpu().numpy()
        assert np.isnan(got_all[:M, N:]).all() and np.isnan(got_all[M:]).all(), "write outside [M, N]"
        got = got_all[:M, :N].astype(np.float64)
        ref = oracle.masked_linear(x, w, s_w, bits, n)["y"]
        rel = F16_REL if out == T.TASQ_OUT_F16 else BF16_REL
        assert np.all(np.abs(got - ref) <= rel * np.abs(ref) + ABS_TINY), (seed, bits)
        if own_status:
            assert int(status.item()) == 0
        else:
            # the call wrote its status bits into the array's own word, which it cleared first
            assert T.tasq_noalloc_device_status(clear=False) == 0


def test_noalloc_size_limit_is_exact(T):
    """The largest token count whose codes fit the fixed array runs (and matches the oracle on a few
    rows); one token more is refused before anything is enqueued."""
    s = torch.cuda.current_stream()
    K, N, n = 16384, 64, 64
    cap = T.TASQ_NOALLOC_SCRATCH_BYTES
    M = cap // K
    while _need(M, K) > cap:
        M -= 1
    assert _need(M + 1, K) > cap
    rng = np.random.default_rng(5)
    x = rng.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    xd, wd, swd = (torch.from_numpy(a).cuda() for a in (x, w, s_w))
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    T.tasq_linear_forward_noalloc(xd, M, K, K, wd, swd, N, 6, n, y, N, T.TASQ_OUT_F16, None, s)
    torch.cuda.synchronize()
    assert T.tasq_noalloc_device_status() == 0
    rows = np.array([0, 1, M // 2, M - 2, M - 1])
    ref = oracle.masked_linear(x[rows], w, s_w, 6, n)["y"]
    got = y[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= F16_REL * np.abs(ref) + ABS_TINY)
    with pytest.raises(T.TasqError) as ei:
        T.tasq_linear_forward_noalloc(xd, M + 1, K, K, wd, swd, N, 6, n, y, N, T.TASQ_OUT_F16, None, s)
    assert ei.value.status == T.TASQ_ERR_WORKSPACE


def test_noalloc_rejects_sizes_beyond_its_fixed_scratch(T):
    K, N, n = 16384, 64, 64
    M = T.TASQ_NOALLOC_SCRATCH_BYTES // K + 1
    x = torch.empty((8, K), dtype=torch.float16, device="cuda")
    w = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty((N,), dtype=torch.float32, device="cuda")
    y = torch.empty((8, N), dtype=torch.float16, device="cuda")
    with pytest.raises(T.TasqError) as ei:
        # sizes are checked before any pointer is used, so the small buffers are never touched
        T.tasq_linear_forward_noalloc(x, M, K, K, w, sw, N, 8, n, y, N, T.TASQ_OUT_F16, None, None)
    assert ei.value.status == T.TASQ_ERR_WORKSPACE
    assert "scratch" in ei.value.message
