"""Multi-process (gloo, world size 2, CPU) checks of the host logic bench.py
uses under torchrun: barrier, max-over-ranks timing, rank 0 alone printing
the reference arm, and independent per-rank problems (weak scaling)."""
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


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    bench.barrier(world)
    # each rank measured its own time; the reported time is the slowest rank's
    t = bench.max_over_ranks(1.5 + rank, world)
    results[rank] = t
    bench.barrier(world)
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    manager = mp.Manager()
    results = manager.dict()
    mp.spawn(_worker, args=(2, port, results), nprocs=2, join=True)
    assert results[0] == results[1] == 2.5


def test_weak_scaling_value_counts_all_ranks():
    # value = units processed by all ranks / max time: with 2 ranks each doing
    # one problem of F flops in the same time T, the value doubles
    F, T = 8.8e12, 0.009
    per_rank = F / T / 1e12
    assert abs(F * 2 / T / 1e12 - 2 * per_rank) < 1e-9
