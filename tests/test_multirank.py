"""The benchmark's multi-rank host logic on two gloo ranks (CPU): the job time
is the slowest rank's time, every rank gets the same value, and the whole-job
throughput counts every replica's bytes.  Decode products shard by output
rows with no exchange, so the N-GPU run is N independent replicas; these are
the only collective steps it takes."""
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


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local = [3.0, 7.5][rank]
        dist.barrier()
        ms = bench.job_time_ms(local, world, torch.device("cpu"))
        gbs = bench.job_throughput_gbs(world, 100, 55_225_344, ms)
        out[rank] = (ms, gbs)
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    ms, gbs = res[0]
    assert ms == 7.5
    assert gbs == pytest.approx(2 * 100 * 55_225_344 / 7.5e-3 / 1e9)


def test_single_rank_is_its_own_time():
    import bench
    assert bench.job_time_ms(4.25, 1, torch.device("cpu")) == 4.25
