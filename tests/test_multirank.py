"""The N > 1 bench path on CPU: two gloo ranks reduce their timed regions to
the slowest one (the whole-job time) and report ms per layer over the layers
all ranks processed; under the reference arm only rank 0 works."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, steps, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q.put((rank, bench.job_time(times[rank], steps, world)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, steps = 2, 5
    times = [100.0, 130.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, steps, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(world))
    for r in range(world):
        total, per_layer = got[r]
        assert total == pytest.approx(130.0)
        assert per_layer == pytest.approx(130.0 / (steps * world))


def test_single_rank_is_its_own_time():
    assert bench.job_time(42.0, 3, 1) == (42.0, 14.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    called = []
    monkeypatch.setattr(bench, "reference_arm", lambda args: called.append(args))
    bench.main()
    assert called == [] and capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    bench.main()
    assert len(called) == 1
