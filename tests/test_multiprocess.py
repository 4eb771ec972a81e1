"""The bench's multi-rank logic on CPU: two gloo ranks, max-over-ranks timing.

On B200s `bench.py --gpus N` runs one independent replica of the layer step per
rank (the path has no exchange step), reduces each rank's CUDA-event time with
a MAX all-reduce and reports units of all ranks / that time.  The same helpers
run here over gloo with CPU tensors.
"""

import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, result_path):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    ms = [3.0, 5.0][rank]
    slowest = bench.max_over_ranks(ms, "cpu")
    value = bench.job_throughput(7.2e12, world, slowest)
    gathered = [None] * world
    dist.all_gather_object(gathered, (rank, slowest, value))
    if rank == 0:
        torch.save(gathered, result_path)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time(tmp_path):
    port = 29500 + (os.getpid() % 1000)
    out = tmp_path / "result.pt"
    mp.start_processes(_worker, args=(2, port, str(out)), nprocs=2, start_method="spawn", join=True)
    results = torch.load(out)
    assert [r[1] for r in results] == [5.0, 5.0]
    assert all(r[2] == pytest.approx(7.2e12 * 2 / 5e-3) for r in results)
