"""The multi-GPU path is independent replicas (sequences never exchange data);
its only cross-rank steps are the barrier and the max-over-ranks timing of
bench.py.  Checked here with two gloo ranks on CPU."""
import datetime
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    dist.barrier()
    t = bench.max_over_ranks(1.5 + rank, world, "cpu")      # rank 1 is the slow one
    rate = bench.whole_job_rate(world, 40, t)
    q.put((rank, t, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_time_is_the_slowest_and_rate_counts_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [2.5, 2.5]          # both ranks see the slowest rank's time
    assert [o[2] for o in out] == [32.0, 32.0]        # 2 ranks x 40 steps / 2.5 s


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    assert bench.whole_job_rate(1, 100, 0.5) == 200.0
