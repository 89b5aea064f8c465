"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, no GPU.

The layer runs as independent replicas (rows of x are independent; no data
exchange), so the only cross-rank logic is the timing reduction: every rank's
step time is reduced with MAX and the whole-job rate counts all ranks' work.
"""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    local = [1.0 + rank, 10.0 - rank, 3.0 * (rank + 1)]       # per-rank step / kernel / e2e ms
    got = bench.max_over_ranks(local, "cpu")
    rate = bench.whole_job_rate(2.0e9, got[0], world)
    out[rank] = (got, rate)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_whole_job_rate(world):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    expect = [1.0 + (world - 1), 10.0, 3.0 * world]
    for rank in range(world):
        got, rate = res[rank]
        assert got == expect
        assert rate == pytest.approx(world * 2.0e9 / (expect[0] * 1e-3))


def test_single_process_is_identity():
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.whole_job_rate(1.0e9, 1.0, 1) == pytest.approx(1.0e12)
