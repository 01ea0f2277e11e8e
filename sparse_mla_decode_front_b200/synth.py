"""Seeded synthetic inputs for the sparse MLA gather-decode block.

This module only *constructs inputs*: shapes, value distributions, paged block
tables, slot rows and gather-index sets of the five workloads the block is
exercised on. It holds none of the block's arithmetic (no normalisation, no
projection, no rotation, no attention) and is imported by both the CUDA path's
tests/bench and the CPU oracle's tests, so the two see identical bytes.

Workloads (DeepSeek-V3.2 MLA shapes; the page "MLA Attention Block Gather
Decode Kernel API Reference" gives the tensor list and their ranks):

  tiny      T=2,   H=256,  Lq=64,   L=64,  dn=32,  dr=16, dv=32,  h=4,   bs=16
  slice16   T=1,   H=7168, Lq=1536, L=512, dn=128, dr=64, dv=128, h=16,  bs=64
  batch32   T=32,  same dims, h=128, contexts U[8192, 32768], P=2048
  gather128 T=128, same dims, h=128, contexts U[32768, 131072], P=2048
  mask64    T=64,  same dims, h=128, contexts log-U[512, 65536], P=4096

Conventions fixed here (they describe the synthetic inputs, not the method):
  * bf16 tensors are numpy ``uint16`` bit patterns, produced by
    round-to-nearest-even of fp32 samples.
  * weights ~ N(0, 1/fan_in); hidden ~ N(0, 1); RMSNorm gammas are fp32
    1 + 0.1 N(0, 1); previously written cache rows are bf16 N(0, 1).
  * a token's position is ``context - 1``; the flat cache row of position p of
    token t is ``block_table[t, p // bs] * bs + p % bs`` (the paged layout of
    ``kv_cache [n_blocks, 1, block_size, kv_row_dim]``), which is how the
    generator places each token's own slot.
  * cos/sin tables: cos(pos * theta^(-2i/dr)) with theta = 10000, built in fp64
    and stored fp32 (the caller-supplied RoPE tables).
  * every block_table entry, including entries past a token's context, names a
    real physical block, so a key that should have been masked still reads
    allocated memory.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

ROPE_THETA = 10000.0


@dataclasses.dataclass(frozen=True)
class Dims:
    n_tokens: int
    hidden: int
    q_lora_rank: int
    kv_lora_rank: int
    qk_nope_head_dim: int
    qk_rope_head_dim: int
    v_head_dim: int
    n_heads: int
    block_size: int
    n_blocks: int
    max_blocks_per_seq: int
    n_prior: int

    @property
    def kv_row_dim(self) -> int:
        return self.kv_lora_rank + self.qk_rope_head_dim

    @property
    def qk_head_dim(self) -> int:
        return self.qk_nope_head_dim + self.qk_rope_head_dim

    def as_tuple(self):
        return dataclasses.astuple(self)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    description: str


WORKLOADS: List[Workload] = [
    Workload("tiny", 0, "T=2 H=256 h=4 L=64 P=32, 4 masked keys per token"),
    Workload("slice16", 1, "T=1 H=7168 h=16 L=512 P=2048, context 4096"),
    Workload("batch32", 2, "T=32 H=7168 h=128 P=2048, contexts U[8192,32768]"),
    Workload("gather128", 3, "T=128 H=7168 h=128 P=2048, contexts U[32768,131072], 1M-row pool"),
    Workload("mask64", 4, "T=64 H=7168 h=128 P=4096, contexts logU[512,65536], masked/future keys, shared blocks"),
]
WORKLOAD_BY_NAME = {w.name: w for w in WORKLOADS}


# ---------------------------------------------------------------------------
# bf16 helpers (storage format conversion of *samples*, not method arithmetic)
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 samples to bf16 (nearest, ties to even); return uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return ((b + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    chunk = 1 << 24
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        v = rng.standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[s:e] = f32_to_bf16_bits(v)
    return out.reshape(shape)


def _gamma(rng: np.random.Generator, n: int) -> np.ndarray:
    return (1.0 + 0.1 * rng.standard_normal(n)).astype(np.float32)


# ---------------------------------------------------------------------------
# Dims per workload
# ---------------------------------------------------------------------------

def _v32_dims(n_tokens, n_heads, block_size, n_blocks, max_blocks, n_prior) -> Dims:
    return Dims(n_tokens=n_tokens, hidden=7168, q_lora_rank=1536, kv_lora_rank=512,
                qk_nope_head_dim=128, qk_rope_head_dim=64, v_head_dim=128,
                n_heads=n_heads, block_size=block_size, n_blocks=n_blocks,
                max_blocks_per_seq=max_blocks, n_prior=n_prior)


def workload_dims(index: int) -> Dims:
    if index == 0:
        return Dims(n_tokens=2, hidden=256, q_lora_rank=64, kv_lora_rank=64,
                    qk_nope_head_dim=32, qk_rope_head_dim=16, v_head_dim=32,
                    n_heads=4, block_size=16, n_blocks=16, max_blocks_per_seq=8,
                    n_prior=32)
    if index == 1:
        return _v32_dims(1, 16, 64, 1024, 64, 2048)
    if index == 2:
        return _v32_dims(32, 128, 64, 65536, 512, 2048)
    if index == 3:
        return _v32_dims(128, 128, 64, 16384, 2048, 2048)
    if index == 4:
        return _v32_dims(64, 128, 64, 65536, 1088, 4096)
    raise ValueError(f"unknown workload index {index}")


# ---------------------------------------------------------------------------
# Index structures
# ---------------------------------------------------------------------------

def _flat_row(block_table: np.ndarray, t: int, p: int, bs: int) -> int:
    return int(block_table[t, p // bs]) * bs + p % bs


def _contexts(index: int, rng: np.random.Generator, T: int) -> np.ndarray:
    if index == 0:
        return np.array([40, 70], dtype=np.int64)
    if index == 1:
        return np.array([4096], dtype=np.int64)
    if index == 2:
        return rng.integers(8192, 32768, size=T, endpoint=True)
    if index == 3:
        return rng.integers(32768, 131072, size=T, endpoint=True)
    if index == 4:
        u = rng.uniform(math.log(512.0), math.log(65536.0), size=T)
        return np.clip(np.floor(np.exp(u)).astype(np.int64), 512, 65536)
    raise ValueError(index)


def _block_tables(index: int, rng: np.random.Generator, d: Dims, ctx: np.ndarray) -> np.ndarray:
    T, bs, nb, mb = d.n_tokens, d.block_size, d.n_blocks, d.max_blocks_per_seq
    bt = np.empty((T, mb), dtype=np.int64)
    if index == 0:
        perm = rng.permutation(nb)
        bt[0] = perm[0:8]
        bt[1] = perm[8:16]
    elif index == 1:
        bt[0] = rng.choice(nb, size=mb, replace=False)
    elif index in (2, 4):
        # In-context logical blocks: disjoint random physical blocks across
        # all sequences. Past-context entries: any block (never dereferenced).
        need = [(int(c) + bs - 1) // bs for c in ctx]
        pool = rng.permutation(nb)
        off = 0
        for t in range(T):
            bt[t, :need[t]] = pool[off:off + need[t]]
            off += need[t]
            bt[t, need[t]:] = rng.integers(0, nb, size=mb - need[t])
        if index == 4:
            # Token pairs (2i, 2i+1) keep their current rows in ONE physical
            # block, at distinct offsets (the caller-side sharing the mask/
            # write-ordering stress case asks for).
            for t in range(0, T - 1, 2):
                pa, pb = int(ctx[t]) - 1, int(ctx[t + 1]) - 1
                bt[t + 1, pb // bs] = bt[t, pa // bs]
    elif index == 3:
        # Pool of 1M rows is smaller than the ~10.5M positions in flight, so
        # blocks are shared across sequences (drawn with replacement), except
        # each token's current block, which is exclusive to it.
        cur = rng.choice(nb, size=T, replace=False)
        is_cur = np.zeros(nb, dtype=bool)
        is_cur[cur] = True
        others = np.flatnonzero(~is_cur)
        bt[:] = others[rng.integers(0, others.size, size=(T, mb))]
        for t in range(T):
            bt[t, (int(ctx[t]) - 1) // bs] = cur[t]
    else:
        raise ValueError(index)
    return bt.astype(np.int32)


def _gather_indices(index: int, rng: np.random.Generator, d: Dims, ctx: np.ndarray) -> np.ndarray:
    T, P = d.n_tokens, d.n_prior
    gi = np.empty((T, P), dtype=np.int64)
    for t in range(T):
        pos = int(ctx[t]) - 1
        if index == 0:
            past = rng.choice(pos + 1, size=P - 4, replace=False)
            fut = pos + 1 + rng.choice(127 - pos, size=4, replace=False)
            sel = np.concatenate([past, fut])
        elif index in (1, 2, 3):
            sel = rng.choice(pos + 1, size=P, replace=False)
        elif index == 4:
            if pos + 1 < P:
                past = np.arange(pos + 1)
                fut = pos + 1 + rng.choice(P, size=P - (pos + 1), replace=False)
            else:
                n_fut = P // 4
                past = rng.choice(pos + 1, size=P - n_fut, replace=False)
                fut = pos + 1 + rng.choice(P, size=n_fut, replace=False)
            sel = np.concatenate([past, fut])
        else:
            raise ValueError(index)
        gi[t] = rng.permutation(sel)
    return gi.astype(np.int32)


def _adjust_pair_offsets(ctx: np.ndarray, bs: int) -> np.ndarray:
    """Make paired tokens' current positions land at distinct block offsets."""
    ctx = ctx.copy()
    for t in range(0, ctx.size - 1, 2):
        if (ctx[t] - 1) % bs == (ctx[t + 1] - 1) % bs:
            ctx[t + 1] += 1 if ctx[t + 1] < 65536 else -1
    return ctx


def rope_tables(positions: np.ndarray, rope_dim: int, theta: float = ROPE_THETA):
    """Caller-side RoPE tables cos/sin [T, rope_dim/2] (fp64 -> fp32)."""
    i = np.arange(rope_dim // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / rope_dim)
    ang = positions.astype(np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


# ---------------------------------------------------------------------------
# Whole input set
# ---------------------------------------------------------------------------

def make_indices(index: int, seed: Optional[int] = None):
    """Index structures of workload ``index`` and the generator state after them.

    Returns (rng, dims, contexts, positions, block_table, gather_indices,
    slot_mapping); ``make_inputs`` continues drawing from the same ``rng``.
    """
    d = workload_dims(index)
    rng = np.random.Generator(np.random.PCG64(1000 + index if seed is None else seed))
    T, bs = d.n_tokens, d.block_size
    ctx = _contexts(index, rng, T)
    if index == 4:
        ctx = _adjust_pair_offsets(ctx, bs)
    positions = (ctx - 1).astype(np.int32)
    block_table = _block_tables(index, rng, d, ctx)
    gather_indices = _gather_indices(index, rng, d, ctx)
    slot_mapping = np.array([_flat_row(block_table, t, int(positions[t]), bs) for t in range(T)],
                            dtype=np.int32)
    return rng, d, ctx, positions, block_table, gather_indices, slot_mapping


def make_inputs(index: int, seed: Optional[int] = None) -> Dict[str, object]:
    """Build the seeded inputs of workload ``index`` (0..4).

    Returns a dict with the block's argument names. bf16 tensors are uint16
    bit arrays, gammas/cos/sin fp32, index tensors int32. ``kv_cache`` is a
    full [n_blocks, 1, block_size, kv_row_dim] uint16 array in which only the
    rows some token may read are filled (the rest are zero pages); the filled
    flat row ids are in ``cache_fill_rows`` so a device copy can be made by
    zero-fill + scatter.
    """
    rng, d, ctx, positions, block_table, gather_indices, slot_mapping = make_indices(index, seed)
    T, H, Lq, L = d.n_tokens, d.hidden, d.q_lora_rank, d.kv_lora_rank
    dn, dr, dv, h, R = d.qk_nope_head_dim, d.qk_rope_head_dim, d.v_head_dim, d.n_heads, d.kv_row_dim
    bs = d.block_size

    # Weights and activations.
    hidden_states = _normal_bf16(rng, (T, H), 1.0)
    input_norm_w = _gamma(rng, H)
    wq_a = _normal_bf16(rng, (H, Lq), 1.0 / math.sqrt(H))
    q_norm_w = _gamma(rng, Lq)
    wq_b = _normal_bf16(rng, (Lq, h * (dn + dr)), 1.0 / math.sqrt(Lq))
    wkv_a = _normal_bf16(rng, (H, R), 1.0 / math.sqrt(H))
    kv_norm_w = _gamma(rng, L)
    q_absorb_w = _normal_bf16(rng, (h, dn, L), 1.0 / math.sqrt(dn))
    out_absorb_w = _normal_bf16(rng, (h, dv, L), 1.0 / math.sqrt(L))
    o_proj_w = _normal_bf16(rng, (h * dv, H), 1.0 / math.sqrt(h * dv))
    cos, sin = rope_tables(positions, dr)

    # Prior cache rows: every row a selected, in-range position refers to.
    rows = set()
    for t in range(T):
        pos = int(positions[t])
        for p in gather_indices[t]:
            p = int(p)
            if 0 <= p <= pos:
                rows.add(_flat_row(block_table, t, p, bs))
    fill = np.array(sorted(rows), dtype=np.int64)
    kv_cache = np.zeros((d.n_blocks, 1, bs, R), dtype=np.uint16)
    flat = kv_cache.reshape(d.n_blocks * bs, R)
    if fill.size:
        flat[fill] = _normal_bf16(rng, (fill.size, R), 1.0)

    return dict(
        dims=d, workload=WORKLOADS[index].name,
        hidden_states=hidden_states, input_norm_w=input_norm_w.reshape(1, H),
        wq_a=wq_a, q_norm_w=q_norm_w.reshape(1, Lq), wq_b=wq_b, wkv_a=wkv_a,
        kv_norm_w=kv_norm_w.reshape(1, L), q_absorb_w=q_absorb_w,
        out_absorb_w=out_absorb_w, o_proj_w=o_proj_w, cos=cos, sin=sin,
        kv_cache=kv_cache, slot_mapping=slot_mapping, block_table=block_table,
        positions=positions, gather_indices=gather_indices,
        n_heads=h, qk_nope_head_dim=dn, qk_rope_head_dim=dr, kv_lora_rank=L,
        softmax_scale=1.0 / math.sqrt(dn + dr), norm_eps=1e-6,
        cache_fill_rows=fill, contexts=ctx.astype(np.int64),
    )


TENSOR_ARGS = ("hidden_states", "input_norm_w", "wq_a", "q_norm_w", "wq_b", "wkv_a",
               "kv_norm_w", "q_absorb_w", "out_absorb_w", "o_proj_w", "cos", "sin",
               "kv_cache", "slot_mapping", "block_table", "positions", "gather_indices")


# ---------------------------------------------------------------------------
# Fused RMSNorm + router top-K inputs (page "RMSNorm Router Top-K A2AV Kernel API
# Reference"): the MoE router that follows the attention block in a DeepSeek-V3
# decoder layer (256 routed experts, 8 per token), plus small and ragged cases.
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class RouterCase:
    name: str
    index: int
    n_tokens: int
    hidden: int
    n_experts: int
    top_k: int
    act: str          # "sigmoid" | "softmax"
    bias: bool
    note: str


ROUTER_CASES: List[RouterCase] = [
    RouterCase("router_tiny", 0, 3, 256, 16, 4, "softmax", True, "T=3 H=256 E=16 K=4 softmax, bias"),
    RouterCase("router_ds128", 1, 128, 7168, 256, 8, "sigmoid", True,
               "T=128 H=7168 E=256 K=8 sigmoid, bias (DeepSeek-V3 routed experts)"),
    RouterCase("router_one", 2, 1, 7168, 64, 6, "sigmoid", False, "T=1 H=7168 E=64 K=6 sigmoid, no bias"),
    RouterCase("router_ragged", 3, 37, 1024, 96, 5, "softmax", True, "T=37 H=1024 E=96 K=5 softmax, bias"),
    RouterCase("router_tall", 4, 300, 1024, 128, 4, "softmax", True,
               "T=300 H=1024 E=128 K=4 softmax, bias (three token tiles, the last ragged)"),
    RouterCase("router_wide", 5, 16, 1024, 512, 8, "sigmoid", True,
               "T=16 H=1024 E=512 K=8 sigmoid, bias (beyond the single launch's 256 experts)"),
    RouterCase("router_odd", 6, 5, 1040, 80, 7, "softmax", True,
               "T=5 H=1040 E=80 K=7 softmax, bias (a partial last K block; experts not a multiple of 32)"),
]
ROUTER_CASE_BY_NAME = {c.name: c for c in ROUTER_CASES}


def make_router_inputs(index: int, seed: Optional[int] = None) -> Dict[str, object]:
    """Seeded inputs of router case ``index``: bf16 bit patterns (uint16) for the
    hidden states [T, H], gamma [H] (1 + 0.1 N(0, 1)), router weights [H, E]
    (N(0, 1/H)) and bias [E] (N(0, 0.1^2), or None); eps 1e-6."""
    c = ROUTER_CASES[index]
    rng = np.random.default_rng(2000 + index if seed is None else seed)
    T, H, E = c.n_tokens, c.hidden, c.n_experts
    return dict(
        case=c,
        hidden_states=_normal_bf16(rng, (T, H), 1.0),
        gamma=f32_to_bf16_bits(_gamma(rng, H)),
        router_weights=_normal_bf16(rng, (H, E), 1.0 / math.sqrt(H)),
        router_bias=_normal_bf16(rng, (E,), 0.1) if c.bias else None,
        eps=1e-6,
        top_k=c.top_k,
        act=c.act,
    )


def make_o_proj_inputs(n_tokens: int, heads_dv: int, hidden: int, seed: int) -> Dict[str, np.ndarray]:
    """Seeded inputs of the o-projection alone, as bf16 bit patterns (uint16): the
    heads' outputs o [T, heads_dv] ~ N(0, 1/4) (the scale of attention contexts
    after out-absorption) and o_proj_w [heads_dv, hidden] ~ N(0, 1/heads_dv)."""
    rng = np.random.default_rng(seed)
    return dict(o=_normal_bf16(rng, (n_tokens, heads_dv), 0.5),
                o_proj_w=_normal_bf16(rng, (heads_dv, hidden), 1.0 / math.sqrt(heads_dv)))
