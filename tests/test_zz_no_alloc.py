"""The allocation-free entry point, tasq_linear_forward_noalloc, against tasq_linear_forward.

Some callers cannot call cudaMalloc: code running inside an allocator callback, hosts that give
all device memory to their own arena, or harnesses that forbid allocation. They call
tasq_linear_forward_noalloc, which takes the weights directly and keeps the activation codes in
a fixed device array inside the library. This file is collected last on purpose, so that a run
stopping at the first failure has already run every other test. It must pass alone in a fresh
process and after the other tests: the fixed array keeps whatever the previous call left there.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

F16_REL = 1e-3
ABS_TINY = 2.0 ** -24


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
    w = rng.integers(-127, 128, size=(N, Kp)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    return x.astype(np.float16), w, s_w


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
