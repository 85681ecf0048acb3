"""The multi-GPU bench path's host logic on CPU: two gloo ranks.

Decode shards by request: every rank owns its own pool, allocator and batch,
and the only cross-rank step is the bench's reduction of timings (max) and
work (sum).  These tests run that reduction and the per-rank workload build
with world_size 2 on the gloo backend.
"""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import paged_kv_cache_354_b200 as pk
    import workloads

    times = [10.0 + rank, 20.0 - rank, 1.5 * (rank + 1)]
    work = [100.0 * (rank + 1), 7.0, 3.0]
    res = bench.combine_ranks(times, work, torch.device("cpu"), world)
    # every rank builds the same per-rank workload state with its own allocator
    p = workloads.plan("llama8b")
    a = pk.PaAlloc(p.num_blocks, p.shape.block_size, p.initial_order)
    ids = workloads.populate(a, p)
    tables, lens = a.block_tables(ids, int(np.max(p.seq_lens)) // p.shape.block_size + 1)
    digest = torch.tensor([float(tables.sum()), float(lens.sum())], dtype=torch.float64)
    gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(gathered, digest)
    out[rank] = (res, [g.tolist() for g in gathered])
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_reduction_and_workloads():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for rank in range(world):
        res, digests = out[rank]
        assert res[:3] == (11.0, 20.0, 3.0)  # max over ranks
        assert res[3:] == (300.0, 14.0, 6.0)  # sum over ranks
        assert digests[0] == digests[1]  # same per-rank state (weak scaling)
