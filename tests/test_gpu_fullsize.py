"""Full-size parity: every distinct layer shape of every workload at its full token count, run
through tasq_linear_forward exactly as the bench launches it, checked on a seeded sample of
token rows (plus the whole last, ragged token tile) against the oracle computed row by row.
Each layer runs at the lowest bit width its schedule gives it and at 8 bits."""
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
    low = [int(sched[j::len(wl.block_layers)].min()) for j in picked]
    table = np.array([[8, b] for b in low], np.uint8)
    s = torch.cuda.current_stream()
    ctx = T.tasq_linear_create(layers, 2, n, M, 0, s)
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
        for step, bits in ((0, 8), (1, low[li])):
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
