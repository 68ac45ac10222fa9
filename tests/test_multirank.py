"""The multi-rank bench path on the CPU: two gloo ranks, the same aggregation the
bench applies to its CUDA-event times under torchrun (replicas: no collective on
the data path, only the max of the per-rank times)."""
import datetime
import os
import socket
import sys
from pathlib import Path

import torch
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, str(ROOT))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    ms = bench.max_over_ranks(1.0 + 2.0 * rank, world, "cpu")     # rank 1 is the slow one
    rate = bench.whole_job_rate(1000.0, world, ms)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    out.put((rank, ms, rate))


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, ms, rate in got:
        assert ms == 3.0
        assert abs(rate - 1000.0 * 2 / 3e-3) < 1e-6


def test_one_rank_needs_no_process_group():
    sys.path.insert(0, str(ROOT))
    import bench
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.whole_job_rate(10.0, 1, 2.0) == 5000.0
