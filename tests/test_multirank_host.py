"""Host logic of bench.py for more than one rank, run on CPU as two gloo processes.

bench.py runs one replica of the whole workload per GPU (the path shards along tokens with no
exchange), so its only cross-rank steps are barriers and the max-over-ranks reduction of the
timed durations; the reference arm runs on rank 0 alone. Both are checked here without a GPU.
"""
import datetime
import json
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, values, queue) -> None:
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(values[rank], dist, "cpu")
        dist.barrier()
        queue.put((rank, got))
    finally:
        dist.destroy_process_group()


def _run_ranks(values):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, len(values), port, values, queue)) for r in range(len(values))]
    for p in procs:
        p.start()
    try:
        out = dict(queue.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    return out


def test_max_over_ranks_with_two_gloo_ranks():
    # rank 1 is the slow one: both ranks must report its time
    assert _run_ranks([3.25, 7.5]) == {0: 7.5, 1: 7.5}


def test_max_over_ranks_without_a_process_group():
    import bench

    assert bench.max_over_ranks(2.0, None, "cpu") == 2.0


def test_reference_arm_prints_nothing_on_other_ranks(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
                       "--workload", "single"]) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
