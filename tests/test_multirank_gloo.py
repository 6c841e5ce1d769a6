"""Multi-rank host logic on CPU with the gloo backend (world size 2): the
bench's job time is the maximum over ranks, its throughput counts every
rank's replica, and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        ws, r, local = bench._dist()
        assert (ws, r, local) == (world, rank, rank)
        mine = 100.0 + 25.0 * rank                      # rank 1 is the slow one
        worst = bench.max_over_ranks(mine)
        value = bench.job_tflops(bench.FLOPS_PER_STEP, 10, world, worst)
        q.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    import bench
    expect = bench.FLOPS_PER_STEP * 10 * world / (125.0e-3) / 1e12
    for rank, worst, value in got:
        assert worst == 125.0
        assert value == pytest.approx(expect)


def test_reference_arm_is_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup = 1, 0
    bench.run_reference(A())                           # must return at once, printing nothing
    assert capsys.readouterr().out == ""
