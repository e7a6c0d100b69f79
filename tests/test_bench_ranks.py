"""The benchmark's multi-rank path on CPU: two gloo ranks, each with its own
timings, agree on the slowest rank's values, and the whole-job throughput
counts every replica's tokens (the layer runs as independent replicas, so
this reduction is the only cross-rank step)."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - 3.0 * rank], world, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_slowest_rank_and_job_throughput():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1] == [2.0, 10.0]
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_tokens_per_s(2, 16384, 2.0) == 2 * 16384 / 2e-3
    assert bench.max_over_ranks([3.0, 4.0], 1, torch.device("cpu")) == [3.0, 4.0]
