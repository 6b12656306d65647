"""The multi-process path of bench.py on CPU: two gloo ranks.

bench.py runs one process per GPU; every rank owns an independent shard of
sequences (weak scaling, no collective on the data path) and the reported
time is the maximum over ranks while the work is the sum. This checks the
rank plumbing that does not need a GPU: the process group, the max/sum
reductions, distinct shards per rank, and that the reference arm leaves
every rank but 0 without work.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    from bit_rotated_kv_block_b200 import workloads

    class A:
        seed = 0
        steps = 1
        warmup = 0
    w_, r_, l_ = bench.dist_setup(A)
    try:
        assert (w_, r_, l_) == (world, rank, rank)
        assert torch.distributed.get_backend() == "gloo"
        bench.barrier(world)
        mx = bench.max_over_ranks(1.5 + rank, world, "cpu")
        sm = bench.sum_over_ranks(10.0 * (rank + 1), world, "cpu")
        w = workloads.llama8b(seed=bench.shard_seed(0, rank), S=2, ctx=32, spare_pages=2)
        k, _, _, _ = w.prefill_tokens()
        ref = bench.run_reference(A, world, rank) if rank != 0 else "skipped"
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.array([mx, sm, float(np.abs(k.astype(np.float64)).sum()),
                          0.0 if ref is None else 1.0]))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r0 = np.load(tmp_path / "r0.npy")
    r1 = np.load(tmp_path / "r1.npy")
    assert r0[0] == r1[0] == 2.5          # max over ranks
    assert r0[1] == r1[1] == 30.0         # sum over ranks
    assert r0[2] != r1[2]                 # each rank draws its own shard
    assert r1[3] == 0.0                   # reference arm: rank 1 does no work
