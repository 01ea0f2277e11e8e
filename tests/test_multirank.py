"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): every rank
builds its own replica batch and the reported time is the max over ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sparse_mla_decode_front_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank]
        out[rank] = bench.max_over_ranks(mine)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        assert out[0] == [11.0, 5.0] and out[1] == [11.0, 5.0]


def test_single_process_identity():
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_replicas_are_distinct_batches():
    assert bench.replica_seed(3, 0) is None
    seeds = {bench.replica_seed(3, r) for r in range(1, 8)}
    assert len(seeds) == 7 and 1003 not in seeds
    a = synth.make_indices(0, seed=bench.replica_seed(0, 0))[5]
    b = synth.make_indices(0, seed=bench.replica_seed(0, 1))[5]
    assert not (a == b).all()
