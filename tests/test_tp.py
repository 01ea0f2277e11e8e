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


# ---------------------------------------------------------------- fused head split

def test_head_split_output_brute_force():
    # Pin: the oracle's head-split sum equals the plain product, written as loops,
    # on tiny shards (3 ranks of 2 heads x 4 value columns, hidden 5).
    rng = np.random.default_rng(11)
    T, world, k, H = 3, 3, 8, 5
    o = [rng.standard_normal((T, k)) for _ in range(world)]
    w = [rng.standard_normal((k, H)) for _ in range(world)]
    y = oracle.head_split_output(o, w)
    for t in range(T):
        for j in range(H):
            acc = 0.0
            for r in range(world):
                for i in range(k):
                    acc += o[r][t, i] * w[r][i, j]
            assert abs(y[t, j] - acc) <= 1e-12 * (1 + abs(acc))


def test_head_split_output_of_block_parts(tiny):
    # Pin: splitting the block's per-head outputs and o_proj_w rows by heads and summing
    # the ranks' o-projections gives the block's output.
    d = tiny["dims"]
    y, _, parts = oracle.block(_fresh(tiny), return_parts=True)
    o = np.stack([p["o"].reshape(-1) for p in parts])
    w = oracle.bf16_to_f64(tiny["o_proj_w"])
    for world in (1, 2, 4):
        cols = d.n_heads // world * d.v_head_dim
        got = oracle.head_split_output([o[:, r * cols:(r + 1) * cols] for r in range(world)],
                                       [w[r * cols:(r + 1) * cols] for r in range(world)])
        np.testing.assert_allclose(got, y, rtol=1e-12, atol=1e-13 * np.abs(y).max())


def _fake_ipc(rank):
    export = lambda t: f"r{rank}:{tuple(t.shape)}:{t.dtype}".encode()
    opened = {}

    def open_(blob):
        opened[blob] = 0x10000 * (len(opened) + 1)
        return opened[blob]
    return export, open_, opened


def _peer_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        export, open_, opened = _fake_ipc(rank)
        closed = []
        pb = tp.PeerBuffers.exchange(rank, world, 4, 256, device="cpu", export=export, open_=open_,
                                     close=closed.append)
        t = pb.table(rank, 7)
        out[rank] = dict(world=t.world, rank=t.rank, epoch=t.epoch,
                         acc=list(t.acc)[:world], out=list(t.out)[:world], flags=list(t.flags)[:world],
                         own=[pb.own[k].data_ptr() for k in ("acc", "out", "flags")],
                         opened={k.decode(): v for k, v in opened.items()},
                         shapes=[tuple(pb.own[k].shape) for k in ("acc", "out", "flags")])
        pb.close()
        out[f"closed{rank}"] = closed
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_peer_buffers_exchange_over_gloo():
    # Host logic of the fused split: each rank allocates its own buffers, trades
    # exports with the group, maps every peer's (a fake mapping here) and lists all
    # ranks' addresses in rank order, its own entries being its own buffers.
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_peer_worker, args=(world, port, out), nprocs=world, join=True)
        for r in range(world):
            o = out[r]
            assert (o["world"], o["rank"], o["epoch"]) == (world, r, 7)
            assert o["shapes"] == [(4, 256 // world), (4, 256), (4,)]
            for i, k in enumerate(("acc", "out", "flags")):
                assert o[k][r] == o["own"][i]
                peer = 1 - r
                name = {"acc": f"r{peer}:(4, {256 // world}):torch.float32", "out": f"r{peer}:(4, 256):torch.bfloat16",
                        "flags": f"r{peer}:(4,):torch.int32"}[k]
                assert o[k][peer] == o["opened"][name]
            assert sorted(out[f"closed{r}"]) == sorted(o["opened"].values())


def test_peer_buffers_local_and_rejections():
    pb = tp.PeerBuffers.local(4, 2, 512, device="cpu")
    t = pb.table(3, 2 ** 32 + 5)
    assert (t.world, t.rank, t.epoch) == (4, 3, 5)   # the epoch counts modulo 2^32
    assert len({t.acc[r] for r in range(4)}) == 4 and t.acc[4] is None
    assert pb.ranks[2]["acc"].shape == (2, 128) and not pb.ranks[2]["flags"].any()
    for world, hidden in [(0, 512), (9, 2304), (4, 500), (3, 96 * 3 + 32)]:
        with pytest.raises(ValueError):
            tp.PeerBuffers(world, 2, hidden, "cpu")


def test_peer_buffers_reset_zeroes_every_local_rank():
    pb = tp.PeerBuffers.local(2, 2, 64, device="cpu")
    for bufs in pb.ranks:
        bufs["acc"].fill_(3.0)
        bufs["flags"].fill_(7)
        bufs["out"].fill_(1.0)
    met = []
    pb.reset(barrier=lambda: met.append(True))
    assert met == [True, True]
    for bufs in pb.ranks:
        assert not bufs["acc"].any() and not bufs["flags"].any()
        assert bufs["out"].eq(1.0).all()   # outputs are the caller's to keep


def test_peer_buffers_reset_drains_before_zeroing():
    # After a timed-out step a late peer may still add into this rank's buffers: every rank
    # first finishes its own GPU's work and meets the others, and only then zeroes; a second
    # meeting keeps anyone from starting the next step before every zero fill has finished.
    pb = tp.PeerBuffers.local(2, 2, 64, device="cpu")
    log = []
    pb.reset(barrier=lambda: log.append("meet"), zero=lambda: log.append("zero"), sync=lambda: log.append("sync"))
    assert log == ["sync", "meet", "zero", "sync", "meet"]


def test_fused_step_epoch_wraps_through_a_reset():
    # The table's epoch is 32 bits and 0 is not a step number: the step that would carry
    # epoch 2^32 first resets the split (all ranks together) and runs as epoch 1.
    class FakeBuffers:
        def __init__(self):
            self.resets, self.epochs = 0, []

        def reset(self, barrier=None):
            self.resets += 1

        def table(self, rank, epoch):
            self.epochs.append(epoch)
            return None

        own = {"out": None}
    step = tp.TPFusedDecodeStep.__new__(tp.TPFusedDecodeStep)
    step.rank, step.world, step.buffers = 0, 2, FakeBuffers()
    step.epoch = 2 ** 32 - 2
    calls = []
    step.step = type("S", (), {"t": {}, "dims": None, "scale": 1.0, "eps": 1e-6, "workspace": None})()
    orig = tp.api.mla_block_gather_decode
    tp.api.mla_block_gather_decode = lambda *a, **k: calls.append(k["tp"])
    try:
        t = {k: None for k in ("hidden_states", "input_norm_w", "wq_a", "q_norm_w", "wq_b", "wkv_a", "kv_norm_w",
                               "q_absorb_w", "out_absorb_w", "o_proj_w", "cos", "sin", "kv_cache",
                               "slot_mapping", "block_table", "positions", "gather_indices")}
        step.step.t = t
        step.run()
        step.run()
    finally:
        tp.api.mla_block_gather_decode = orig
    assert step.buffers.epochs == [2 ** 32 - 1, 1] and step.buffers.resets == 1 and step.epoch == 1


def test_peer_buffers_exchange_unmaps_on_failure():
    # A mapping that fails part-way: the handles mapped before it are closed again.
    gathered = [{k: f"r{r}{k}".encode() for k in ("acc", "out", "flags")} for r in range(3)]
    opened, closed = [], []

    def open_(blob):
        if blob == b"r2acc":
            raise RuntimeError("peer mapping refused")
        opened.append(len(opened) + 1)
        return opened[-1]
    with pytest.raises(RuntimeError, match="refused"):
        tp.PeerBuffers.exchange(0, 3, 2, 96, device="cpu", export=lambda t: b"", open_=open_,
                                close=closed.append, all_gather=lambda mine: gathered)
    assert sorted(closed) == opened == [1, 2, 3]
