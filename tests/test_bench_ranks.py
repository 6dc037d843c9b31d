"""Host logic of `bench.py --gpus N` on the CPU: world-size-2 gloo ranks.

The step does not shard (each rank is an independent replica), so the only multi-rank logic is
the timing: every rank's time is reduced to the slowest rank's, and the whole-job throughput is
N x steps over that time.  The reference arm runs on rank 0 only.
"""
import datetime
import os
import socket

import pytest


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.0, 5.0, 4.0, 1.0][rank]  # each rank's own timed region
        slowest = bench.max_over_ranks(ms, dist, "cpu")
        value = bench.replica_throughput(world, 10, slowest)
        dist.barrier()
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_replicas_report_the_slowest_rank(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(world))
    expect_ms = max([3.0, 5.0, 4.0, 1.0][:world])
    for rank, slowest, value in got:
        assert slowest == expect_ms, (rank, slowest)
        assert value == pytest.approx(world * 10 / (expect_ms / 1e3)), (rank, value)


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(2.5, None, "cpu") == 2.5
    assert bench.replica_throughput(1, 4, 2.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    assert bench.run_reference(bench.parse()) is None
    assert capsys.readouterr().out == ""  # no work and no line on the other ranks
