"""Data-parallel replicas on CPU: world_size 2 over gloo.  Each rank takes
its shard of the batch (libnle's shard plan), computes its outputs (here the
oracle stands in for the device kernels, since this host has no GPU), and
the gathered result must equal the whole batch computed at once."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from chunked_block_self_b200 import dp, nle
        from chunked_block_self_b200 import workloads as wl
        x = wl.block_inputs(lengths=[230, 17, 401, 0, 199, 88, 600], heads=2, seed=21)
        bounds = nle.nle_shard_plan_host(x["lengths"], world, 200)
        a, b, local_cu = dp.local_shard(x["cu"], bounds, rank)
        o = oracle.block_attn(x["q"][a:b], x["k"][a:b], x["v"][a:b], local_cu, n_threads=1)
        t = torch.zeros(x["total"], 2, 64, dtype=torch.float64)
        t[a:b] = torch.from_numpy(o)
        dist.all_reduce(t)      # disjoint row ranges: the sum is the gather
        if rank == 0:
            full = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], n_threads=1)
            np.save(result_path, np.abs(t.numpy() - full).max())
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_reassemble(tmp_path):
    world, port = 2, _free_port()
    path = str(tmp_path / "diff.npy")
    mp.start_processes(_worker, args=(world, port, path), nprocs=world, start_method="spawn")
    assert float(np.load(path)) == 0.0
