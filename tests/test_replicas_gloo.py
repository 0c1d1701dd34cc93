"""Host-side logic of the multi-GPU bench (replicas, no data-path collective): a world-size-2
gloo job on the CPU checks the barrier and the max / sum over ranks that turn per-rank timings
into the job's time and throughput."""
import os
import socket
import sys
from pathlib import Path

import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, str(ROOT))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    bench.barrier(world)
    ms = 10.0 + 5.0 * rank          # per-rank timed region (ms)
    tokens = 8 * 64                  # per-rank tokens
    out[rank] = (bench.max_over_ranks(ms, world), bench.sum_over_ranks(tokens, world))
    bench.barrier(world)
    dist.destroy_process_group()


def test_replicas_max_time_and_total_tokens():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        assert out[r] == (15.0, 1024.0)
    # whole-job throughput = all ranks' tokens / slowest rank's time
    assert out[0][1] / (out[0][0] / 1e3) == 1024 / 0.015
