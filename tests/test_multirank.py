"""Multi-rank host logic of bench.py on CPU: two gloo ranks reduce their
step times (maximum over ranks), emitted tokens and kernel launches (sums
over ranks) the way the N-GPU benchmark does; the aggregate throughput is
whole-job tokens over the slowest rank's time."""
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        times = [1.0 + rank, 10.0 - rank, 0.5 * (rank + 1)]   # step, e2e, lm (ms)
        tokens = 3 + 2 * rank
        got, total, launches = bench.reduce_over_ranks(times, tokens, world, "cpu", 12 * (rank + 1))
        assert got == [float(world), 10.0, 0.5 * world], got
        assert total == sum(3 + 2 * r for r in range(world)), total
        assert launches == sum(12 * (r + 1) for r in range(world)), launches
        # every rank sees the same whole-job figures
        value = total / (got[0] / 1e3)
        assert abs(value - 8 / 2e-3) < 1e-6 if world == 2 else True
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_like_the_benchmark():
    mp.spawn(_rank, args=(2, _free_port()), nprocs=2, join=True)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    got, total, launches = bench.reduce_over_ranks([1.5, 2.5], 7, 1, "cpu", 24000)
    assert got == [1.5, 2.5] and total == 7 and launches == 24000
