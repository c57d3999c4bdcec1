"""The N > 1 host path of bench.py on CPU: two gloo ranks, as torchrun would
start them (one replica of the workload per rank, no data-path collective;
only the timing is combined, as the maximum over ranks)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import sys
    import torch
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    # each rank times its own replica; the job's time is the slowest rank's
    ms = bench._max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
    rate = bench.whole_job_rate(1000, ms, world)
    # the reference arm runs on rank 0 only; the other ranks return without work
    class A:
        steps, warmup = 1, 0
    ref = bench.run_reference(A(), rank, world) if rank != 0 else "skipped on rank 0"
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    out.put((rank, ms, rate, ref))


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate, ref in res:
        assert ms == pytest.approx(15.0)            # max over ranks
        assert rate == pytest.approx(2 * 1000 / 0.015)  # whole job: both replicas' units
    assert res[1][3] is None                           # rank 1 does no reference work
