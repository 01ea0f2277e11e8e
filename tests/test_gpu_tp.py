"""Tensor parallelism over heads on one GPU.

* Partials: the ranks of a world of 2 run one after the other on the same device
  (no rank waits on another), each writing its fp32 partial
  (mla_launch_opts.out_f32); their sum, rounded once to bf16, meets the block's
  bar against the fp64 oracle and agrees with the all-heads call.
* Fused reduction (include/mla_tp.h): every rank of a world of 1, 2, 4 or 8 runs
  on this GPU inside one launch of each kernel (n_local = world), so the ranks'
  waits on one another are satisfied within one cooperative launch; every rank's
  output is compared element by element with the oracle's head-split sum.
* CUDA IPC: a second process on the same GPU maps the first one's output buffer
  and writes the fused op's result into it (no process waits on a kernel of the
  other)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_mla_decode_front_b200 import _lib, api, synth, tp
from sparse_mla_decode_front_b200.device import DecodeStep, _to_torch
from test_gpu_parity import OUT_TOL, oracle_run

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl,tokens", [(0, None), (2, [0, 13, 31])])
def test_head_shards_on_one_gpu(wl, tokens):
    inp = synth.make_inputs(wl)
    world = 2
    ranks = [tp.TPDecodeStep(inp, r, world) for r in range(world)]
    total = sum(rk.partial().clone() for rk in ranks)
    torch.cuda.synchronize()
    assert all(rk.device_status() == 0 for rk in ranks)
    y = total.to(torch.bfloat16).float().cpu().numpy().astype(np.float64)
    y_ref, _ = oracle_run(inp, tokens)
    sel = slice(None) if tokens is None else list(tokens)
    assert np.abs(y[sel] - y_ref).max() / np.abs(y_ref).max() <= OUT_TOL
    full = DecodeStep(inp).run().float()
    torch.cuda.synchronize()
    y_full = full.cpu().numpy().astype(np.float64)
    assert np.abs(y - y_full).max() <= 2.0 ** -7 * np.abs(y_full).max()


# ---------------------------------------------------------------- fused head split

# A bf16 store of an fp32 sum: half a bf16 step of |y| (2^-9 relative) plus the fp32
# accumulation error of the split sums, bounded by 2^-16 of the largest output.
def _close_to_bf16_of(y_gpu: np.ndarray, y_ref: np.ndarray) -> np.ndarray:
    return np.abs(y_gpu - y_ref) <= 2.0 ** -8 * np.abs(y_ref) + 2.0 ** -16 * np.abs(y_ref).max()


def _bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


# (2, 16, 1024, 384) and (1, 5, 512, 640): an odd count of 128-feature tiles, so the last CTA
# tile of the paired projection holds one feature tile and one past the hidden size
@pytest.mark.parametrize("world,T,heads_dv,hidden", [(1, 37, 1024, 512), (2, 128, 4096, 2048),
                                                     (4, 1, 2048, 1024), (8, 128, 16384, 7168),
                                                     (8, 77, 4096, 2048), (2, 16, 1024, 384),
                                                     (1, 5, 512, 640)])
def test_fused_o_proj_reduction_all_ranks_on_one_gpu(world, T, heads_dv, hidden):
    k = heads_dv // world
    pb = tp.PeerBuffers.local(world, T, hidden)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    counts = []
    for epoch in (1, 2):   # the second step checks the zeroed accumulators and the epoch counts
        x = synth.make_o_proj_inputs(T, heads_dv, hidden, seed=7000 + 10 * world + epoch)
        o, w = _to_torch(x["o"], True).cuda(), _to_torch(x["o_proj_w"], True).cuda()
        api.mla_tp_o_proj_allreduce(o, w, pb.table(0, epoch), world, ws)
        torch.cuda.synchronize()
        status = int(ws[:4].view(torch.int32).item())
        assert status == 0, f"device status {status:#x}"
        of, wf = oracle.bf16_to_f64(x["o"]), oracle.bf16_to_f64(x["o_proj_w"])
        y_ref = oracle.head_split_output([of[:, r * k:(r + 1) * k] for r in range(world)],
                                         [wf[r * k:(r + 1) * k] for r in range(world)])
        outs = [pb.ranks[r]["out"] for r in range(world)]
        ok = _close_to_bf16_of(_bf16_host(outs[0]), y_ref)
        assert ok.all(), f"{(~ok).sum()} elements off, first at {np.argwhere(~ok)[:3]}"
        for r in range(1, world):   # every rank holds the same rounded sums
            assert torch.equal(outs[r].view(torch.int16), outs[0].view(torch.int16))
        for r in range(world):
            assert not pb.ranks[r]["acc"].any(), "accumulator not left zero"
        counts.append([pb.ranks[r]["flags"][:2].tolist() for r in range(world)])
    for r in range(world):   # counters grow by the same count every step, a multiple of world
        assert counts[1][r][0] == 2 * counts[0][r][0] > 0 and counts[0][r][0] % world == 0
        assert counts[1][r][1] == 2 * counts[0][r][1] > 0 and counts[0][r][1] % world == 0


def test_fused_reduction_wait_runs_out_then_reset_recovers():
    # The failure form a bounded device wait allows: a table whose epoch is ahead of the
    # counters (what a rank that missed a step would see), so the finish kernel's waits
    # run out after their limit; the kernel sets MLA_DEV_WAIT_TIMEOUT in the status word
    # and returns, and the context stays usable. reset() brings the accumulators and
    # counters back, and the next step (epoch 1) is right again.
    world, T, heads_dv, hidden = 2, 16, 1024, 512
    k = heads_dv // world
    pb = tp.PeerBuffers.local(world, T, hidden)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    x = synth.make_o_proj_inputs(T, heads_dv, hidden, seed=7300)
    o, w = _to_torch(x["o"], True).cuda(), _to_torch(x["o_proj_w"], True).cuda()
    api.mla_tp_o_proj_allreduce(o, w, pb.table(0, 5), world, ws)
    torch.cuda.synchronize()
    status = int(ws[:4].view(torch.int32).item())
    assert status & _lib.MLA_DEV_WAIT_TIMEOUT, f"device status {status:#x}"
    pb.reset()
    ws.zero_()
    api.mla_tp_o_proj_allreduce(o, w, pb.table(0, 1), world, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    of, wf = oracle.bf16_to_f64(x["o"]), oracle.bf16_to_f64(x["o_proj_w"])
    y_ref = oracle.head_split_output([of[:, r * k:(r + 1) * k] for r in range(world)],
                                     [wf[r * k:(r + 1) * k] for r in range(world)])
    for r in range(world):
        ok = _close_to_bf16_of(_bf16_host(pb.ranks[r]["out"]), y_ref)
        assert ok.all(), f"rank {r}: {(~ok).sum()} elements off"
        assert not pb.ranks[r]["acc"].any()


@pytest.mark.parametrize("wl", [0, 2])
def test_fused_block_world_of_one(wl):
    # The block call with a one-rank peer table: the o-projection reduces into the
    # table's accumulator and the finish kernel writes the output; same bar as the
    # plain call, and agreement with it.
    inp = synth.make_inputs(wl)
    step = DecodeStep(inp)
    d = step.dims
    pb = tp.PeerBuffers.local(1, d.n_tokens, d.hidden)
    t = step.t
    for epoch in (1, 2):
        n = api.mla_block_gather_decode(
            t["hidden_states"], t["input_norm_w"], t["wq_a"], t["q_norm_w"], t["wq_b"], t["wkv_a"],
            t["kv_norm_w"], t["q_absorb_w"], t["out_absorb_w"], t["o_proj_w"], t["cos"], t["sin"],
            t["kv_cache"], t["slot_mapping"], t["block_table"], t["positions"], t["gather_indices"],
            None, d, step.scale, step.eps, step.workspace, None, tp=pb.table(0, epoch))
        torch.cuda.synchronize()
        assert step.device_status() == 0
    y = _bf16_host(pb.own["out"])
    y_ref, _ = oracle_run(inp)
    assert np.abs(y - y_ref).max() / np.abs(y_ref).max() <= OUT_TOL
    plain = _bf16_host(DecodeStep(inp).run())
    assert np.abs(y - plain).max() <= 2.0 ** -7 * np.abs(plain).max()
    assert not pb.own["acc"].any()


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _ipc_worker(rank, port, T, heads_dv, hidden, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        torch.cuda.set_device(0)
        if rank == 0:   # owns the output buffer; the other process writes into it
            y = torch.zeros(T, hidden, dtype=torch.bfloat16, device="cuda")
            torch.cuda.synchronize()
            dist.broadcast_object_list([api.mla_ipc_export(y)], src=0)
            dist.barrier()   # the writer has finished and unmapped
            out["y"] = y.float().cpu().numpy()
        else:
            blob = [None]
            dist.broadcast_object_list(blob, src=0)
            addr = api.mla_ipc_open(blob[0])
            x = synth.make_o_proj_inputs(T, heads_dv, hidden, seed=7100)
            o, w = _to_torch(x["o"], True).cuda(), _to_torch(x["o_proj_w"], True).cuda()
            pb = tp.PeerBuffers.local(1, T, hidden)
            pb.addr["out"][0] = addr
            ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
            api.mla_tp_o_proj_allreduce(o, w, pb.table(0, 1), 1, ws)
            torch.cuda.synchronize()
            out["status"] = int(ws[:4].view(torch.int32).item())
            api.mla_ipc_close(addr)
            dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ipc_mapping_between_two_processes():
    T, heads_dv, hidden = 16, 1024, 512
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_ipc_worker, args=(_free_port(), T, heads_dv, hidden, out), nprocs=2, join=True)
        assert out["status"] == 0
        x = synth.make_o_proj_inputs(T, heads_dv, hidden, seed=7100)
        y_ref = oracle.o_projection(oracle.bf16_to_f64(x["o"]), oracle.bf16_to_f64(x["o_proj_w"]))
        ok = _close_to_bf16_of(out["y"].astype(np.float64), y_ref)
        assert ok.all()
