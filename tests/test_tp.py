"""Tensor parallelism over heads (sparse_mla_decode_front_b200/tp.py) on CPU: the
head shards' partial outputs sum to the all-heads output (the oracle's head
linearity, page "MLA Attention Block Gather Decode Kernel API Reference": the
output is "this rank's" partial, o_proj rows by head), and the reduction plumbing
sums the ranks' fp32 partials over a world-size-2 gloo group."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_mla_decode_front_b200 import synth, tp


def _fresh(inp):
    out = dict(inp)
    out["kv_cache"] = inp["kv_cache"].copy()
    return out


@pytest.fixture(scope="module")
def tiny():
    return synth.make_inputs(0)


@pytest.mark.parametrize("world", [2, 4])
def test_head_shards_sum_to_the_full_block(tiny, world):
    y = oracle.block(_fresh(tiny))
    total = sum(oracle.block(_fresh(tp.head_shard(tiny, r, world))) for r in range(world))
    np.testing.assert_allclose(total, y, rtol=1e-12, atol=1e-13 * np.abs(y).max())


def test_head_shard_slices_and_rejections(tiny):
    d = tiny["dims"]
    s = tp.head_shard(tiny, 1, 2)
    qk = d.qk_nope_head_dim + d.qk_rope_head_dim
    assert s["dims"].n_heads == d.n_heads // 2
    np.testing.assert_array_equal(s["wq_b"], tiny["wq_b"][:, 2 * qk:4 * qk])
    np.testing.assert_array_equal(s["o_proj_w"], tiny["o_proj_w"][2 * d.v_head_dim:4 * d.v_head_dim])
    assert s["kv_cache"] is tiny["kv_cache"] and s["wq_a"] is tiny["wq_a"]   # replicated
    for rank, world in [(0, 3), (2, 2), (-1, 2), (0, 0)]:
        with pytest.raises(ValueError):
            tp.head_shard(tiny, rank, world)


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = synth.make_inputs(0)
        part = torch.from_numpy(oracle.block(_fresh(tp.head_shard(inp, rank, world))).astype(np.float32))
        out[rank] = tp.reduce_partials(part).numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_partials_over_gloo(tiny):
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        y = oracle.block(_fresh(tiny))
        for r in range(world):
            np.testing.assert_allclose(out[r], y, rtol=1e-5, atol=1e-6 * np.abs(y).max())
