"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, each with its
own timing; the job's time is the slowest rank's and the rate counts the
units of every rank (weak scaling, no data-path collective)."""
import os
import socket
import sys
from pathlib import Path

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    my_ms = [3.0, 5.0][rank]
    ms_max = bench.max_over_ranks(my_ms)
    bench.barrier()
    rate = bench.whole_job_rate(32, world, ms_max)
    out[rank] = (ms_max, rate)
    dist.destroy_process_group()


def test_two_rank_timing_aggregation():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms_max, rate = res[rank]
        assert ms_max == 5.0
        assert abs(rate - 2 * 32 / 5e-3) < 1e-6


def test_single_process_is_identity():
    sys.path.insert(0, str(ROOT))
    import bench
    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.whole_job_rate(32, 1, 2.0) == 16000.0
