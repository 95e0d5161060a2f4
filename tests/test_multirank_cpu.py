"""The benchmark's multi-process path on CPU: two gloo ranks stand in for
two GPUs.  Each rank runs the full per-GPU workload (weak scaling); the
only collectives are the timing barrier and the MAX of the elapsed times,
and the reference arm runs on rank 0 alone."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, elapsed, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK="0")
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms = bench.max_over_ranks(elapsed[rank], "cpu")
    rate = bench.job_rate(world, 1000.0, ms)
    # the reference arm: rank 0 times the oracle, every other rank returns at once
    ran = None
    if rank != 0:
        ran = bench.run_reference(None, None) is None
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, rate, bench.rank_env(), ran))


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    elapsed = [12.5, 20.0]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, elapsed, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    for rank, ms, rate, env, ran in results:
        assert ms == 20.0                        # the slower rank's time
        assert rate == pytest.approx(2 * 1000.0 / 0.020)
        assert env == (2, rank, 0)
    assert results[1][4] is True                 # rank 1 skipped the reference arm


def test_one_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_rate(1, 10.0, 1000.0) == 10.0
