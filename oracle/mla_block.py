"""CPU fp64 oracle for one sparse MLA gather-decode block step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
execute this module; only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` use it. It shares no code,
tables or constants with the CUDA path.

What it computes follows the page "MLA Attention Block Gather Decode Kernel API
Reference" (AWS Neuron NKI library, ``mla_attention_block_gather_decode``),
section "API Reference", one ``:param`` entry per argument. The page prints no
equations; every step below restates a parameter description, and where the
page is open the plainest reading is taken and named in the docstring.

Precision: inputs are read exactly from their bf16 / fp32 storage and every
operation is fp64. The one rounding the method itself fixes is the cache write:
``kv_cache`` is bf16 storage, so the row written at ``slot_mapping[t]`` is the
fp64 row rounded once, to nearest-even bf16, and the attention reads that
stored row back.

Pins (tests/test_oracle_pins.py) tie every function here to facts fixed
outside this file: a hand-derived worked case, the absorbed == unabsorbed
identity against torch's fp64 scaled_dot_product_attention, full-prefix ==
dense attention, invariance to gather order / masked entries / physical block
relabelling, softmax closed forms, RMSNorm scale invariance, RoPE rotation
properties, head linearity and the bf16 rounding rule.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np


# ---------------------------------------------------------------------------
# Storage conversions
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as fp64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values once to bf16 (nearest, ties to even); uint16 bits.

    bf16 keeps 8 significant bits and fp32's exponent range. With
    x = m * 2**e, 0.5 <= |m| < 1 (frexp), the spacing of bf16 values in x's
    binade is 2**(e - 8), floored at the subnormal spacing 2**-133.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ue = np.maximum(e - 8, -133)
    q = np.rint(np.ldexp(x, -ue))          # rint: round half to even
    v = np.ldexp(q, ue)                    # exactly representable in bf16
    with np.errstate(over="ignore"):
        f = v.astype(np.float32)           # exact (or +-inf past the range)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Elementary steps
# ---------------------------------------------------------------------------

def rmsnorm(v: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: v / sqrt(mean(v^2) + eps) * gamma.

    ``input_norm_w``, ``q_norm_w`` and ``kv_norm_w`` are plain gammas (the
    page lists them as fp32 RMSNorm gammas, no ``1 + gamma`` offset); one
    ``norm_eps`` serves every RMSNorm of the front-fold (:param norm_eps).
    """
    ms = np.mean(v * v, axis=-1, keepdims=True)
    return v / np.sqrt(ms + eps) * gamma


def rope_interleaved(v: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Interleaved RoPE over the last axis (width dr), tables of width dr/2.

    "Interleaved" (:param cos, sin) is read as rotating adjacent pairs
    (2i, 2i+1) by the angle whose cosine/sine are cos[i], sin[i]:
        out[2i]   = v[2i] cos_i - v[2i+1] sin_i
        out[2i+1] = v[2i] sin_i + v[2i+1] cos_i
    """
    a = v[..., 0::2]
    b = v[..., 1::2]
    out = np.empty_like(v)
    out[..., 0::2] = a * cos - b * sin
    out[..., 1::2] = a * sin + b * cos
    return out


def resolve_row(block_table_row: np.ndarray, position: int, p: int, block_size: int) -> int:
    """Map a selected absolute position to a flat cache row, or -1 if masked.

    :param positions: the causal mask compares each selected key with the
    token's own position; a key is kept iff 0 <= p <= position (p == position
    is the row this step writes). :param block_table: the per-sequence
    logical-to-physical block map resolves the kept position to
    block_table[p // block_size] * block_size + p % block_size.
    """
    if p < 0 or p > position:
        return -1
    return int(block_table_row[p // block_size]) * block_size + p % block_size


def softmax(s: np.ndarray) -> np.ndarray:
    """Softmax over the last axis (max-shifted, fp64)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


# ---------------------------------------------------------------------------
# Front-fold (mla_decode_qkv) per token
# ---------------------------------------------------------------------------

class _F64Inputs:
    """fp64 views of the block's inputs (exact conversions of the storage)."""

    def __init__(self, inp: Dict[str, object]):
        d = inp["dims"]
        self.d = d
        self.hidden = bf16_to_f64(inp["hidden_states"])
        self.g_in = np.asarray(inp["input_norm_w"], np.float64).reshape(-1)
        self.wq_a = bf16_to_f64(inp["wq_a"])
        self.g_q = np.asarray(inp["q_norm_w"], np.float64).reshape(-1)
        self.wq_b = bf16_to_f64(inp["wq_b"])
        self.wkv_a = bf16_to_f64(inp["wkv_a"])
        self.g_kv = np.asarray(inp["kv_norm_w"], np.float64).reshape(-1)
        self.q_absorb = bf16_to_f64(inp["q_absorb_w"])
        self.out_absorb = bf16_to_f64(inp["out_absorb_w"])
        self.o_proj = bf16_to_f64(inp["o_proj_w"])
        self.cos = np.asarray(inp["cos"], np.float64)
        self.sin = np.asarray(inp["sin"], np.float64)
        self.eps = float(inp["norm_eps"])
        self.scale = float(inp["softmax_scale"])


def input_norm(f: _F64Inputs, t: int) -> np.ndarray:
    """:param input_norm_w -- RMSNorm of the layer input, folded into the front-fold."""
    return rmsnorm(f.hidden[t], f.g_in, f.eps)


def kv_row(f: _F64Inputs, t: int) -> np.ndarray:
    """The cache row this token writes, [kv_lora_rank + qk_rope_head_dim], fp64.

    :param wkv_a emits one row per token; the row is read as
    [latent (kv_lora_rank) | k_pe (qk_rope_head_dim)] (kv_lora_rank is "the
    latent width of a cache row"). :param kv_norm_w normalises the latent part
    only (its gamma is [1, kv_lora_rank]); k_pe is rotated with this token's
    cos/sin and stored rotated.
    """
    L = f.d.kv_lora_rank
    kv = input_norm(f, t) @ f.wkv_a
    c = rmsnorm(kv[:L], f.g_kv, f.eps)
    k_pe = rope_interleaved(kv[L:], f.cos[t], f.sin[t])
    return np.concatenate([c, k_pe])


def query_heads(f: _F64Inputs, t: int):
    """Per-head query pieces (q_nope [h, dn], q_pe rotated [h, dr]).

    :param wq_a / q_norm_w / wq_b: q = rmsnorm(xn wq_a, q_norm_w) wq_b, whose
    columns are "every head's [q_nope | q_pe] concatenated", i.e. head-major
    blocks of width dn + dr, nope first.
    """
    d = f.d
    q_a = input_norm(f, t) @ f.wq_a
    q = rmsnorm(q_a, f.g_q, f.eps) @ f.wq_b
    q = q.reshape(d.n_heads, d.qk_nope_head_dim + d.qk_rope_head_dim)
    q_nope = q[:, :d.qk_nope_head_dim]
    q_pe = rope_interleaved(q[:, d.qk_nope_head_dim:], f.cos[t], f.sin[t])
    return q_nope, q_pe


def absorb_query(f: _F64Inputs, q_nope: np.ndarray) -> np.ndarray:
    """:param q_absorb_w [h, dn, L]: map each head's nope query into latent space.

    q_lat[h] = q_nope[h] @ q_absorb_w[h]   ([dn] x [dn, L] -> [L]).
    """
    return np.einsum("hd,hdl->hl", q_nope, f.q_absorb)


# ---------------------------------------------------------------------------
# Core (mla_decode_attention) per token
# ---------------------------------------------------------------------------

def attend_token(f: _F64Inputs, cache_rows_f64: np.ndarray, q_lat: np.ndarray,
                 q_pe: np.ndarray) -> np.ndarray:
    """Latent attention of one token over its kept rows; returns o [h, dv].

    Scores: scale * (q_lat[h] . row[:L] + q_pe[h] . row[L:]) for every kept
    row (all heads share the rows: one latent "KV head"). Softmax over the kept
    rows; the latent part of each row is the value; :param out_absorb_w maps the
    latent context back to the head's value width:
        o[h] = out_absorb_w[h] @ ctx[h]   ([dv, L] x [L] -> [dv]).
    A token with no kept row attends to nothing: ctx = 0, so o = 0.
    """
    d = f.d
    L = d.kv_lora_rank
    if cache_rows_f64.shape[0] == 0:
        return np.zeros((d.n_heads, d.v_head_dim))
    s = f.scale * (q_lat @ cache_rows_f64[:, :L].T + q_pe @ cache_rows_f64[:, L:].T)
    w = softmax(s)
    ctx = w @ cache_rows_f64[:, :L]
    return np.einsum("hvl,hl->hv", f.out_absorb, ctx)


# ---------------------------------------------------------------------------
# The o-projection and its split over heads
# ---------------------------------------------------------------------------

def o_projection(o: np.ndarray, o_proj_w: np.ndarray) -> np.ndarray:
    """:param o_proj_w: y = o @ o_proj_w for o [T, heads * v_head_dim] (the heads'
    outputs side by side) and o_proj_w [heads * v_head_dim, hidden], fp64."""
    return o @ o_proj_w


def head_split_output(o_parts: Sequence[np.ndarray], w_parts: Sequence[np.ndarray]) -> np.ndarray:
    """The introduction's "this rank's" output under a split of the heads over
    ranks: rank r holds its heads' columns of o and their rows of o_proj_w, and
    the block output is the sum over ranks of the partial o-projections."""
    y = None
    for o, w in zip(o_parts, w_parts):
        part = o_projection(o, w)
        y = part if y is None else y + part
    return y


# ---------------------------------------------------------------------------
# The whole block
# ---------------------------------------------------------------------------

def block(inp: Dict[str, object], tokens: Optional[Sequence[int]] = None,
          kv_cache: Optional[np.ndarray] = None, return_parts: bool = False):
    """One decode step: returns y [T, hidden] fp64 (rows of ``tokens`` only if given).

    Order (:param kv_cache -- "the front-fold writes this step's row, and the
    core reads the selected prior rows back"): every token's row is written to
    the cache first, rounded to bf16; then each token attends over its kept
    selected rows, read back from the bf16 cache, so a row written this step
    (the token's own, or another token's in a shared block) is seen.
    :param o_proj_w: y[t] = concat_h(o[t, h]) @ o_proj_w -- this rank's partial
    block output, no residual added.

    ``kv_cache`` (uint16 bits, [n_blocks, 1, block_size, kv_row_dim]) is
    mutated in place; it defaults to ``inp['kv_cache']``.
    """
    f = _F64Inputs(inp)
    d = f.d
    T = d.n_tokens
    cache = inp["kv_cache"] if kv_cache is None else kv_cache
    flat = cache.reshape(d.n_blocks * d.block_size, d.kv_row_dim)
    slot = np.asarray(inp["slot_mapping"])
    bt = np.asarray(inp["block_table"])
    pos = np.asarray(inp["positions"])
    gi = np.asarray(inp["gather_indices"])

    written = np.empty((T, d.kv_row_dim), dtype=np.uint16)
    for t in range(T):
        written[t] = f64_to_bf16(kv_row(f, t))
    for t in range(T):
        flat[int(slot[t])] = written[t]

    sel = list(range(T)) if tokens is None else [int(t) for t in tokens]
    y = np.zeros((len(sel), d.hidden))
    parts = []
    for i, t in enumerate(sel):
        rows = [resolve_row(bt[t], int(pos[t]), int(p), d.block_size) for p in gi[t]]
        rows = [r for r in rows if r >= 0]
        kept = bf16_to_f64(flat[np.array(rows, dtype=np.int64)]) if rows else \
            np.zeros((0, d.kv_row_dim))
        q_nope, q_pe = query_heads(f, t)
        q_lat = absorb_query(f, q_nope)
        o = attend_token(f, kept, q_lat, q_pe)
        y[i] = o.reshape(-1) @ f.o_proj
        if return_parts:
            parts.append(dict(q_nope=q_nope, q_pe=q_pe, q_lat=q_lat, rows=rows, o=o))
    if return_parts:
        return y, written, parts
    return y
