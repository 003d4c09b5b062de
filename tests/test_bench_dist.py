"""The benchmark's multi-process plumbing on CPU: world size 2 over gloo
(max-over-ranks timing, barrier, rank/world discovery from the environment)."""
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
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    bench.init_dist(w, "gloo")
    bench.barrier(w)
    got = bench.reduce_max(1.5 + rank, w, torch.device("cpu"))
    weak_tokens = 2 * 4096 * w      # every rank runs its own copy of the workload
    out[rank] = (got, weak_tokens)
    dist.destroy_process_group()


def test_two_rank_max_and_barrier():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1] == (2.5, 2 * 4096 * 2)


def test_single_process_needs_no_group():
    import bench
    assert bench.reduce_max(3.0, 1, torch.device("cpu")) == 3.0
    bench.barrier(1)
