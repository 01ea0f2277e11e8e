"""Tensor parallelism over heads for the block step (page "MLA Attention Block
Gather Decode Kernel API Reference": the output is "this rank's" attention-block
output; :param n_heads, o_proj_w).

Rank r of a world of W holds heads [r h/W, (r + 1) h/W): the columns of wq_b for
those heads, their q_absorb_w and out_absorb_w slices and their rows of o_proj_w.
Everything else (the down-projections, the norms, the latent cache, the index
tensors) is replicated; every rank writes the same, head-independent, cache rows
into its own replica. Each rank's block call writes its partial output in fp32
(``out_f32``); an all-reduce (NCCL over NVLink between GPUs) sums the partials and
the sum is rounded once to bf16. The o-projection is linear in the heads, so the
sum is the all-heads block output.

The fused form (``PeerBuffers``, ``TPFusedDecodeStep``; include/mla_tp.h) does the
sum inside the o-projection instead: each finished fp32 tile is reduced straight
into the accumulator of the rank owning its hidden columns (a peer GPU's memory
over NVLink), the owner rounds its columns once and writes them into every rank's
output, and two arrival counters per rank order the steps. The peers' buffers are
mapped with CUDA IPC (``mla_ipc_export`` / ``mla_ipc_open``), the handles traded
with an all-gather of the process group.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional

import numpy as np
import torch

from . import _lib, api
from .device import DecodeStep


def head_shard(inp: Dict[str, object], rank: int, world: int) -> Dict[str, object]:
    """Rank ``rank``'s inputs (the seeded-input dict layout): its heads' slices of
    wq_b, q_absorb_w, out_absorb_w and o_proj_w, every other input shared."""
    d = inp["dims"]
    if world < 1 or not 0 <= rank < world or d.n_heads % world:
        raise ValueError(f"{d.n_heads} heads do not split over {world} ranks")
    hl = d.n_heads // world
    h0 = rank * hl
    qk = d.qk_nope_head_dim + d.qk_rope_head_dim
    out = dict(inp)
    out["dims"] = type(d)(**{**d.__dict__, "n_heads": hl})
    out["wq_b"] = np.ascontiguousarray(inp["wq_b"][:, h0 * qk:(h0 + hl) * qk])
    out["q_absorb_w"] = np.ascontiguousarray(inp["q_absorb_w"][h0:h0 + hl])
    out["out_absorb_w"] = np.ascontiguousarray(inp["out_absorb_w"][h0:h0 + hl])
    out["o_proj_w"] = np.ascontiguousarray(inp["o_proj_w"][h0 * d.v_head_dim:(h0 + hl) * d.v_head_dim])
    return out


def reduce_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' fp32 partial outputs in place (all-reduce) and return the sum."""
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(partial, op=torch.distributed.ReduceOp.SUM, group=group)
    return partial


class TPDecodeStep:
    """One rank's share of the block step: its head shard resident on ``device``."""

    def __init__(self, inp: Dict[str, object], rank: int, world: int, device="cuda", group=None):
        self.rank, self.world, self.group = rank, world, group
        self.step = DecodeStep(head_shard(inp, rank, world), device=device)
        d = self.step.dims
        self.partial_f32 = torch.empty((d.n_tokens, d.hidden), dtype=torch.float32, device=self.step.device)

    def partial(self, stream=None) -> torch.Tensor:
        """This rank's fp32 partial output (its heads' share of the o-projection)."""
        s, t = self.step, self.step.t
        api.mla_block_gather_decode(
            t["hidden_states"], t["input_norm_w"], t["wq_a"], t["q_norm_w"], t["wq_b"], t["wkv_a"],
            t["kv_norm_w"], t["q_absorb_w"], t["out_absorb_w"], t["o_proj_w"], t["cos"], t["sin"],
            t["kv_cache"], t["slot_mapping"], t["block_table"], t["positions"], t["gather_indices"],
            None, s.dims, s.scale, s.eps, s.workspace, stream, out_f32=self.partial_f32)
        return self.partial_f32

    def run(self, stream=None) -> torch.Tensor:
        """The all-heads block output (bf16): this rank's partial summed over the group."""
        p = self.partial(stream)
        return reduce_partials(p, self.group).to(torch.bfloat16)

    def device_status(self, stream=None) -> int:
        return self.step.device_status(stream)


_BUFFERS = ("acc", "out", "flags")


class PeerBuffers:
    """The buffers of a head split as one rank sees them: its own accumulator
    [T, hidden / world] fp32, output [T, hidden] bf16 and arrival counters (zeroed
    once), and the addresses of every rank's three buffers (``addr[name][r]``).

    ``exchange`` maps the peers' buffers through CUDA IPC; ``local`` keeps every
    rank's buffers on one device (all ranks computed there, n_local = world)."""

    def __init__(self, world: int, n_tokens: int, hidden: int, device, alloc=None):
        if not 1 <= world <= _lib.MLA_TP_MAX_WORLD or hidden % (32 * world):
            raise ValueError(f"hidden {hidden} does not split into {world} shards of 32-column blocks")
        alloc = alloc or (lambda shape, dtype: torch.zeros(shape, dtype=dtype, device=device))
        self.world, self.n_tokens, self.hidden = world, n_tokens, hidden
        self._alloc = alloc
        self.own = self._new()
        self.addr: Dict[str, List[int]] = {k: [0] * world for k in _BUFFERS}
        self.opened: List[int] = []
        self._close = None

    def _new(self) -> Dict[str, torch.Tensor]:
        return {"acc": self._alloc((self.n_tokens, self.hidden // self.world), torch.float32),
                "out": self._alloc((self.n_tokens, self.hidden), torch.bfloat16),
                "flags": self._alloc((4,), torch.int32)}   # two counters, padded to 16 bytes

    @classmethod
    def local(cls, world: int, n_tokens: int, hidden: int, device="cuda", alloc=None) -> "PeerBuffers":
        pb = cls(world, n_tokens, hidden, device, alloc)
        pb.ranks = [pb.own] + [pb._new() for _ in range(world - 1)]
        for r, bufs in enumerate(pb.ranks):
            for k in _BUFFERS:
                pb.addr[k][r] = bufs[k].data_ptr()
        return pb

    @classmethod
    def exchange(cls, rank: int, world: int, n_tokens: int, hidden: int, device="cuda", group=None,
                 alloc=None, export: Callable = None, open_: Callable = None, close: Callable = None,
                 all_gather: Callable = None) -> "PeerBuffers":
        """Allocate this rank's buffers, trade IPC exports with the group and map the
        peers' buffers (the callables default to the library's IPC calls and
        torch.distributed.all_gather_object)."""
        export = export or api.mla_ipc_export
        open_ = open_ or api.mla_ipc_open
        pb = cls(world, n_tokens, hidden, device, alloc)
        pb._close = close or api.mla_ipc_close
        pb._sync()   # the zero fill has run before any peer can add into these buffers
        mine = {k: export(pb.own[k]) for k in _BUFFERS}
        if all_gather is None:
            gathered = [None] * world
            torch.distributed.all_gather_object(gathered, mine, group=group)
        else:
            gathered = all_gather(mine)
        if len(gathered) != world:
            raise RuntimeError(f"{len(gathered)} ranks answered, expected {world}")
        try:
            for r in range(world):
                for k in _BUFFERS:
                    if r == rank:
                        pb.addr[k][r] = pb.own[k].data_ptr()
                    else:
                        a = open_(gathered[r][k])
                        pb.opened.append(a)
                        pb.addr[k][r] = a
        except Exception:
            pb.close()   # unmap what was mapped before the failure
            raise
        return pb

    def table(self, rank: int, epoch: int) -> "_lib.MlaTpPeers":
        t = _lib.MlaTpPeers()
        t.world, t.rank, t.epoch = self.world, rank, epoch & 0xFFFFFFFF
        for r in range(self.world):
            t.acc[r], t.out[r], t.flags[r] = self.addr["acc"][r], self.addr["out"][r], self.addr["flags"][r]
        return t

    def _sync(self) -> None:
        if self.own["acc"].is_cuda:
            torch.cuda.synchronize(self.own["acc"].device)

    def reset(self, barrier: Optional[Callable] = None, zero: Optional[Callable] = None,
              sync: Optional[Callable] = None) -> None:
        """Zero this rank's accumulator and counters again (every rank does, e.g. after a
        step reported MLA_DEV_WAIT_TIMEOUT) so that the next step's epoch restarts at 1.

        Order: finish this GPU's work, meet the other ranks, zero, finish the zero fill,
        meet again. After a step that timed out, a late peer's projection may still be
        adding into this rank's accumulator and counters; the first meeting waits until
        every rank's GPU has drained (each synchronised its own device before it), so no
        such add can land after the zero fill; the second one keeps every rank from
        starting the next step before all buffers are zero. ``barrier`` defaults to
        torch.distributed.barrier when a group is up; ``zero`` and ``sync`` (the zero fill
        and the device synchronisation) are parameters so the order can be checked
        without a GPU."""
        meet = barrier
        if meet is None and torch.distributed.is_available() and torch.distributed.is_initialized():
            meet = torch.distributed.barrier
        sync = sync or self._sync
        zero = zero or self._zero
        sync()
        if meet is not None:
            meet()
        zero()
        sync()
        if meet is not None:
            meet()

    def _zero(self) -> None:
        for k in ("acc", "flags"):
            self.own[k].zero_()
        for bufs in getattr(self, "ranks", [])[1:]:   # every rank on this device
            for k in ("acc", "flags"):
                bufs[k].zero_()

    def close(self) -> None:
        """Unmap the peers' buffers (after this GPU's work on them has finished)."""
        if self.opened:
            self._sync()
        for a in self.opened:
            self._close(a)
        self.opened = []


class TPFusedDecodeStep:
    """One rank's block step with the o-projection reduced over peer memory: its
    head shard resident on ``device``, the split's buffers mapped through IPC."""

    def __init__(self, inp: Dict[str, object], rank: int, world: int, device="cuda", group=None):
        self.rank, self.world = rank, world
        self.step = DecodeStep(head_shard(inp, rank, world), device=device)
        d = self.step.dims
        self.buffers = PeerBuffers.exchange(rank, world, d.n_tokens, d.hidden, self.step.device, group)
        self.epoch = 0

    def run(self, stream=None) -> torch.Tensor:
        """Enqueue one step; returns this rank's output buffer, which holds the
        all-heads bf16 block output once the step has run."""
        s, t = self.step, self.step.t
        if (self.epoch + 1) & 0xFFFFFFFF == 0:
            # The table's epoch is 32 bits and 0 is not a step number: every rank reaches this
            # step together (same count), brings the counters back to zero and starts again.
            self.reset()
        self.epoch += 1
        api.mla_block_gather_decode(
            t["hidden_states"], t["input_norm_w"], t["wq_a"], t["q_norm_w"], t["wq_b"], t["wkv_a"],
            t["kv_norm_w"], t["q_absorb_w"], t["out_absorb_w"], t["o_proj_w"], t["cos"], t["sin"],
            t["kv_cache"], t["slot_mapping"], t["block_table"], t["positions"], t["gather_indices"],
            None, s.dims, s.scale, s.eps, s.workspace, stream, tp=self.buffers.table(self.rank, self.epoch))
        return self.buffers.own["out"]

    def device_status(self, stream=None) -> int:
        return self.step.device_status(stream)

    def reset(self, barrier: Optional[Callable] = None) -> None:
        """Bring the split's counters and accumulators back to their first-step state
        (all ranks call it together)."""
        self.buffers.reset(barrier)
        self.epoch = 0

    def close(self) -> None:
        self.buffers.close()
