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
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import api
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
