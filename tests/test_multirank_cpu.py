"""The N>1 bench path on CPU: two gloo ranks, max-over-ranks timing and the
whole-job value (every rank's bytes over the slowest rank's time)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench

    local = 10.0 + 5.0 * rank  # rank 1 is the slow one
    mx = bench.max_over_ranks(local, dist, torch.device("cpu"))
    val = bench.whole_job_gbs(world, 1e9, 4, mx)
    dist.barrier()
    dist.destroy_process_group()
    results[rank] = (mx, val)


def test_two_gloo_ranks_take_the_slowest_rank():
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        mx, val = results[r]
        assert mx == 15.0
        # 2 ranks x 1 GB x 4 steps in 15 ms
        assert val == pytest.approx(2 * 1e9 * 4 / 15e-3 / 1e9)


def test_single_rank_needs_no_group():
    import bench

    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
