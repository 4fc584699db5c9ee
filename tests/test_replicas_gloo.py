"""The multi-rank plumbing of bench.py (replicas only: one frame per rank, max-over-ranks
timing, whole-job throughput) with two gloo ranks on CPU."""
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
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ws, r, _ = bench.dist_env()
    assert (ws, r) == (world, rank)
    bench.barrier()
    step_ms = 10.0 + 5.0 * rank                        # rank 1 is the slow one
    ms = bench.reduce_max(step_ms, torch.device("cpu"))
    edges = 1000
    out[rank] = (ms, edges * ws / (ms * 1e-3))
    bench.barrier()
    dist.destroy_process_group()


def test_two_rank_max_timing_and_whole_job_value():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1]
    ms, value = out[0]
    assert ms == 15.0
    assert value == pytest.approx(2 * 1000 / 0.015)
