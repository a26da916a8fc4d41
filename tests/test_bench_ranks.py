"""The multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

With N GPUs the benchmark runs N independent layer solves (weak scaling, no
data-path collective); the step time is the maximum over ranks and the job
throughput counts every rank's layer.
"""
import os
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, q):
    import torch.distributed as tdist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.reduce_max(10.0 + 5.0 * rank, True, "cpu")
        q.put((rank, ms, bench.job_throughput(world, 1000, ms)))
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_step_time_is_max_over_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    slowest = 10.0 + 5.0 * (world - 1)
    for rank, ms, thr in got:
        assert ms == slowest
        assert thr == pytest.approx(world * 1000 / (slowest / 1e3))


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25, False, "cpu") == 3.25
    assert bench.job_throughput(1, 16777216, 11.0) == pytest.approx(16777216 / 0.011)
