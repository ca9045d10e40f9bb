"""The N > 1 path of bench.py: one process per GPU running an independent replica of the
workload (the attention of a chunk needs nothing from other GPUs, so there is no data-path
collective). What the ranks share is host logic: the step time is the max over ranks, the
job's rate counts every replica's units, and only rank 0 reports. Run here as two gloo ranks on
CPU (127.0.0.1)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        env = bench.dist_env()
        t = bench.max_over_ranks(5.0 + 3.0 * rank)      # rank 1 is the slow replica
        t2 = bench.max_over_ranks(9.0 - rank)           # same order of calls on every rank
        rate = bench.job_throughput(world, 32768, t)
        q.put((rank, env, t, t2, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_and_count_every_replica():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, env, t, t2, rate in res:
        assert env == (rank, 2, rank)
        assert t == 8.0 and t2 == 9.0
        assert rate == pytest.approx(2 * 32768 / 8e-3)


def test_without_a_process_group_the_value_is_local():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 100, 50.0) == pytest.approx(2000.0)


def test_reference_arm_on_a_non_zero_rank_exits_without_work(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
