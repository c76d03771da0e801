"""The N > 1 host path of the benchmark on CPU: two gloo ranks take the
slowest rank's time and report the whole job's throughput (replicas only:
the GEMV path has no data-path collective)."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.join(os.path.dirname(__file__), "..")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        ms = bench.max_over_ranks(1.5 + rank, dist)  # rank 1 is the slow one
        out[rank] = ms
        out[world + rank] = bench.job_throughput(world, 1e9, ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world = 2
    out = torch.zeros(2 * world, dtype=torch.float64).share_memory_()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 2.5
    # 2 replicas x 1 GB in 2.5 ms
    assert abs(out[2] - 2 * 1e9 / 2.5e-3 / 1e9) < 1e-9 and out[2] == out[3]


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.job_throughput(1, 2e9, 1.0) == 2000.0
