"""The benchmark's multi-rank host logic on CPU: world size 2 over gloo.

Every rank times its own shard of sequences (weak scaling, no collective on
the data path); the job's time is the slowest rank's, reached by a MAX
all-reduce that every rank takes part in, and the job's rate counts the
units of all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = [3.0, 5.0][rank]                      # this rank's device time (ms)
        slowest = bench.max_over_ranks(mine, dist, "cpu")
        rate = bench.whole_job_rate(world, 1000, 10, slowest)
        out[rank] = (slowest, rate)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_the_job_rate():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        codes = [p.exitcode for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        assert codes == [0, 0], codes
        for r in range(2):
            slowest, rate = out[r]
            assert slowest == 5.0
            assert rate == pytest.approx(2 * 1000 * 10 / 5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(2.5, None, "cpu") == 2.5
    assert bench.whole_job_rate(1, 100, 4, 2.0) == pytest.approx(100 * 4 / 2e-3)
    assert torch.get_default_dtype() == torch.float32
