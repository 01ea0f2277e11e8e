"""Pins of the CPU fp64 oracle to facts fixed outside it.

Each test ties the oracle to something it cannot agree with by construction:
a hand-derived worked case, a library routine (torch's fp64
scaled_dot_product_attention, torch's fp32->bf16 rounding) on an equivalent
but differently written formulation, closed forms, and invariances of the
method. ``test_planted_mistakes_are_caught`` plants plausible mistakes in the
oracle (on the CPU) and checks that the pins fail for each.
"""
import copy
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_block as M
from sparse_mla_decode_front_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def hand_inputs():
    with open(os.path.join(GOLDEN, "hand_case.json")) as fh:
        g = json.load(fh)
    d = synth.Dims(**g["dims"])
    gi = g["inputs"]
    bf = lambda v: synth.f32_to_bf16_bits(np.asarray(v, np.float32))
    cache = np.zeros((d.n_blocks, 1, d.block_size, d.kv_row_dim), np.uint16)
    flat = cache.reshape(-1, d.kv_row_dim)
    for r, v in gi["kv_cache_rows"].items():
        flat[int(r)] = bf(v)
    inp = dict(
        dims=d, hidden_states=bf(gi["hidden_states"]),
        input_norm_w=np.asarray(gi["input_norm_w"], np.float32), wq_a=bf(gi["wq_a"]),
        q_norm_w=np.asarray(gi["q_norm_w"], np.float32), wq_b=bf(gi["wq_b"]),
        wkv_a=bf(gi["wkv_a"]), kv_norm_w=np.asarray(gi["kv_norm_w"], np.float32),
        q_absorb_w=bf(gi["q_absorb_w"]), out_absorb_w=bf(gi["out_absorb_w"]),
        o_proj_w=bf(gi["o_proj_w"]), cos=np.asarray(gi["cos"], np.float32),
        sin=np.asarray(gi["sin"], np.float32), kv_cache=cache,
        slot_mapping=np.asarray(gi["slot_mapping"], np.int32),
        block_table=np.asarray(gi["block_table"], np.int32),
        positions=np.asarray(gi["positions"], np.int32),
        gather_indices=np.asarray(gi["gather_indices"], np.int32),
        softmax_scale=math.log(3.0), norm_eps=float(gi["norm_eps"]))
    return inp, g["expected"]


def fresh(inp):
    out = dict(inp)
    out["kv_cache"] = inp["kv_cache"].copy()
    return out


@pytest.fixture(scope="module")
def tiny():
    return synth.make_inputs(0)


def run(inp, **kw):
    return M.block(fresh(inp), **kw)


# ---------------------------------------------------------------------------
# worked case
# ---------------------------------------------------------------------------

def check_hand_case():
    inp, exp = hand_inputs()
    x = fresh(inp)
    y, written, parts = M.block(x, return_parts=True)
    flat = x["kv_cache"].reshape(-1, inp["dims"].kv_row_dim)
    np.testing.assert_allclose(y, np.asarray(exp["out"], float), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(
        M.bf16_to_f64(flat[exp["written_row_slot"]]), np.asarray(exp["written_row"], float))
    np.testing.assert_array_equal(M.bf16_to_f64(written[0]), np.asarray(exp["written_row"], float))
    np.testing.assert_allclose(parts[0]["q_nope"], exp["q_nope"], atol=1e-15)
    np.testing.assert_allclose(parts[0]["q_pe"], exp["q_pe"], atol=1e-15)
    np.testing.assert_allclose(parts[0]["q_lat"], exp["q_lat"], atol=1e-15)
    assert parts[0]["rows"] == exp["kept_rows"]


def test_hand_case():
    check_hand_case()


# ---------------------------------------------------------------------------
# bf16 rounding of the cache write
# ---------------------------------------------------------------------------

def test_bf16_rounding_ties_and_torch():
    one = 1.0
    cases = {
        one: 0x3F80,
        one + 2.0 ** -8: 0x3F80,                    # tie -> even (1.0)
        one + 3 * 2.0 ** -8: 0x3F82,                # tie -> even (1 + 2^-6)
        one + 2.0 ** -8 + 2.0 ** -30: 0x3F81,       # just above the tie
        -(one + 2.0 ** -8 + 2.0 ** -30): 0xBF81,
        0.0: 0x0000,
        2.0 ** -133: 0x0001,                        # smallest bf16 subnormal
        1.5 * 2.0 ** -133: 0x0002,                  # tie between 1 and 2 -> even
    }
    for v, bits in cases.items():
        assert int(M.f64_to_bf16(np.array([v]))[0]) == bits, (v, hex(bits))
    # Against torch's fp32 -> bf16 (round-to-nearest-even) on fp32 values,
    # where a single rounding from fp64 equals torch's single rounding.
    rng = np.random.default_rng(7)
    x32 = (rng.standard_normal(100000) * np.exp(rng.uniform(-30, 30, 100000))).astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(M.f64_to_bf16(x32.astype(np.float64)), ref)
    # bf16 -> f64 is exact: round trip.
    bits = rng.integers(0, 0x7F80, 5000, dtype=np.uint16)
    np.testing.assert_array_equal(M.f64_to_bf16(M.bf16_to_f64(bits)), bits)


# ---------------------------------------------------------------------------
# absorbed == unabsorbed, against torch's fp64 SDPA
# ---------------------------------------------------------------------------

def test_absorbed_equals_unabsorbed_sdpa(tiny):
    inp = fresh(tiny)
    d = inp["dims"]
    y, _, parts = M.block(inp, return_parts=True)
    flat = inp["kv_cache"].reshape(-1, d.kv_row_dim)
    L = d.kv_lora_rank
    qa = M.bf16_to_f64(tiny["q_absorb_w"])     # [h, dn, L]
    oa = M.bf16_to_f64(tiny["out_absorb_w"])   # [h, dv, L]
    op = M.bf16_to_f64(tiny["o_proj_w"])
    for t in range(d.n_tokens):
        rows = M.bf16_to_f64(flat[np.array(parts[t]["rows"])])
        c, kpe = rows[:, :L], rows[:, L:]
        o = np.zeros((d.n_heads, d.v_head_dim))
        for h in range(d.n_heads):
            # Unabsorbed per-head keys/values: K_nope = c q_absorb_w[h]^T,
            # V = c out_absorb_w[h]^T, K = [K_nope | k_pe].
            k = np.concatenate([c @ qa[h].T, kpe], axis=1)
            v = c @ oa[h].T
            q = np.concatenate([parts[t]["q_nope"][h], parts[t]["q_pe"][h]])
            out = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q)[None, None, None, :], torch.from_numpy(k)[None, None],
                torch.from_numpy(v)[None, None], scale=tiny["softmax_scale"])
            o[h] = out[0, 0, 0].numpy()
        yt = o.reshape(-1) @ op
        np.testing.assert_allclose(y[t], yt, rtol=1e-11, atol=1e-12 * np.abs(yt).max())


# ---------------------------------------------------------------------------
# gather / mask / paging
# ---------------------------------------------------------------------------

def _single_token(inp, t):
    """Sub-problem of token t alone (its own row, tables and indices)."""
    d = inp["dims"]
    x = fresh(inp)
    for k in ("hidden_states", "cos", "sin", "slot_mapping", "block_table", "positions",
              "gather_indices"):
        x[k] = np.ascontiguousarray(inp[k][t:t + 1])
    x["dims"] = synth.Dims(**{**d.__dict__, "n_tokens": 1})
    return x


def test_full_prefix_equals_dense_attention(tiny):
    # Identity block table: position p lives at flat row p. gather_indices is
    # a shuffled [0..pos]; the result must equal dense attention over the
    # first pos+1 rows of the cache in order (torch fp64 SDPA).
    d = tiny["dims"]
    x = _single_token(tiny, 1)
    pos = int(x["positions"][0])
    x["block_table"] = np.arange(d.max_blocks_per_seq, dtype=np.int32)[None, :]
    x["slot_mapping"] = np.array([pos], np.int32)
    rng = np.random.default_rng(3)
    x["gather_indices"] = rng.permutation(pos + 1).astype(np.int32)[None, :]
    x["dims"] = synth.Dims(**{**x["dims"].__dict__, "n_prior": pos + 1})
    cache = x["kv_cache"].reshape(-1, d.kv_row_dim)
    cache[:pos] = synth.f32_to_bf16_bits(rng.standard_normal((pos, d.kv_row_dim)).astype(np.float32))
    y, _, parts = M.block(x, return_parts=True)
    L = d.kv_lora_rank
    rows = M.bf16_to_f64(cache[:pos + 1])
    q = np.concatenate([parts[0]["q_lat"], parts[0]["q_pe"]], axis=1)       # [h, R]
    ctx = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(rows)[None, None].expand(1, d.n_heads, -1, -1),
        torch.from_numpy(rows[:, :L])[None, None].expand(1, d.n_heads, -1, -1),
        scale=tiny["softmax_scale"])[0, :, 0].numpy()                        # [h, L]
    o = np.einsum("hvl,hl->hv", M.bf16_to_f64(tiny["out_absorb_w"]), ctx)
    yd = o.reshape(-1) @ M.bf16_to_f64(tiny["o_proj_w"])
    np.testing.assert_allclose(y[0], yd, rtol=1e-11, atol=1e-12 * np.abs(yd).max())


def test_gather_order_invariance(tiny):
    y = run(tiny)
    x = dict(tiny)
    rng = np.random.default_rng(11)
    x["gather_indices"] = np.stack([rng.permutation(r) for r in tiny["gather_indices"]]).astype(np.int32)
    np.testing.assert_allclose(run(x), y, rtol=1e-13, atol=1e-14)


def test_masked_entries_do_not_matter(tiny):
    d = tiny["dims"]
    y = run(tiny)
    pos = tiny["positions"]
    gi = tiny["gather_indices"]
    # (a) replace every masked entry by another future position / a negative one
    x = dict(tiny)
    g2 = gi.copy()
    for t in range(d.n_tokens):
        m = g2[t] > pos[t]
        g2[t, m] = np.where(np.arange(m.sum()) % 2 == 0, pos[t] + 1, -5)
    x["gather_indices"] = g2
    np.testing.assert_allclose(run(x), y, rtol=1e-13, atol=1e-14)
    # (b) delete the masked entries (fewer prior keys)
    x = dict(tiny)
    keep = [gi[t][gi[t] <= pos[t]] for t in range(d.n_tokens)]
    n = min(k.size for k in keep)
    x["gather_indices"] = np.stack([k[:n] for k in keep]).astype(np.int32)
    x["dims"] = synth.Dims(**{**d.__dict__, "n_prior": n})
    ys = run(x)
    # token whose kept list was cut must differ; the other must match
    for t in range(d.n_tokens):
        if keep[t].size == n:
            np.testing.assert_allclose(ys[t], y[t], rtol=1e-13, atol=1e-14)


def test_block_relabel_invariance(tiny):
    # Moving physical blocks (cache contents together with the tables that
    # point at them) must not change the result.
    d = tiny["dims"]
    y = run(tiny)
    sigma = np.random.default_rng(5).permutation(d.n_blocks)
    x = dict(tiny)
    cache = np.empty_like(tiny["kv_cache"])
    cache[sigma] = tiny["kv_cache"]
    x["kv_cache"] = cache
    x["block_table"] = sigma[tiny["block_table"]].astype(np.int32)
    s = tiny["slot_mapping"]
    x["slot_mapping"] = (sigma[s // d.block_size] * d.block_size + s % d.block_size).astype(np.int32)
    np.testing.assert_allclose(run(x), y, rtol=1e-13, atol=1e-14)


def test_cross_token_write_is_seen(tiny):
    # Two tokens keep their current rows in one physical block at distinct
    # offsets; the token with the larger offset selects the position that maps
    # to the other token's slot. Its result must equal a call in which that
    # row was already in the cache before the step (writes precede reads).
    d = tiny["dims"]
    bs = d.block_size
    x = fresh(tiny)
    pos = [int(p) for p in x["positions"]]
    r, w = (0, 1) if pos[0] % bs > pos[1] % bs else (1, 0)
    assert pos[r] % bs != pos[w] % bs
    bt = x["block_table"].copy()
    bt[r, pos[r] // bs] = bt[w, pos[w] // bs]
    x["block_table"] = bt
    slot = x["slot_mapping"].copy()
    slot[r] = bt[r, pos[r] // bs] * bs + pos[r] % bs
    x["slot_mapping"] = slot
    g = x["gather_indices"].copy()
    g[r, 0] = pos[r] - pos[r] % bs + pos[w] % bs
    x["gather_indices"] = g
    y1, written, parts = M.block(x, return_parts=True)
    assert int(slot[w]) in parts[r]["rows"]
    x2 = fresh(x)
    x2["kv_cache"].reshape(-1, d.kv_row_dim)[int(slot[w])] = written[w]
    np.testing.assert_allclose(M.block(x2), y1, rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------------------
# softmax closed forms
# ---------------------------------------------------------------------------

def _rows_for(inp, t, y_parts):
    d = inp["dims"]
    flat = inp["kv_cache"].reshape(-1, d.kv_row_dim)
    return M.bf16_to_f64(flat[np.array(y_parts[t]["rows"])])


def test_single_valid_key_closed_form(tiny):
    d = tiny["dims"]
    x = fresh(tiny)
    pos = x["positions"]
    g = x["gather_indices"].copy()
    for t in range(d.n_tokens):
        valid = np.flatnonzero(g[t] <= pos[t])
        g[t, valid[1:]] = pos[t] + 1 + (np.arange(valid.size - 1) % (127 - pos[t]))
    x["gather_indices"] = g
    y, _, parts = M.block(x, return_parts=True)
    oa = M.bf16_to_f64(tiny["out_absorb_w"])
    op = M.bf16_to_f64(tiny["o_proj_w"]).reshape(d.n_heads, d.v_head_dim, d.hidden)
    for t in range(d.n_tokens):
        assert len(parts[t]["rows"]) == 1
        c = _rows_for(x, t, parts)[0, :d.kv_lora_rank]
        # one key: weight 1, o[h] = out_absorb_w[h] c, y = sum_h o[h] o_proj[h]
        yc = sum((oa[h] @ c) @ op[h] for h in range(d.n_heads))
        np.testing.assert_allclose(y[t], yc, rtol=1e-12, atol=1e-13)


def test_zero_query_gives_mean_of_latents(tiny):
    d = tiny["dims"]
    x = fresh(tiny)
    x["wq_b"] = np.zeros_like(tiny["wq_b"])
    y, _, parts = M.block(x, return_parts=True)
    oa = M.bf16_to_f64(tiny["out_absorb_w"])
    op = M.bf16_to_f64(tiny["o_proj_w"]).reshape(d.n_heads, d.v_head_dim, d.hidden)
    for t in range(d.n_tokens):
        cbar = _rows_for(x, t, parts)[:, :d.kv_lora_rank].mean(axis=0)
        yc = sum((oa[h] @ cbar) @ op[h] for h in range(d.n_heads))
        np.testing.assert_allclose(y[t], yc, rtol=1e-12, atol=1e-13)


def test_no_valid_key_gives_zero(tiny):
    x = dict(tiny)
    x["gather_indices"] = np.full_like(tiny["gather_indices"], 127)
    x["gather_indices"][0, :3] = -1
    np.testing.assert_array_equal(run(x), 0.0)


# ---------------------------------------------------------------------------
# RMSNorm and RoPE
# ---------------------------------------------------------------------------

def test_rmsnorm_scale_invariance(tiny):
    x = dict(tiny, norm_eps=0.0)
    y, w = M.block(fresh(x), return_parts=True)[:2]
    x2 = dict(x)
    x2["hidden_states"] = synth.f32_to_bf16_bits(2.0 * synth.bf16_bits_to_f32(tiny["hidden_states"]))
    y2, w2 = M.block(fresh(x2), return_parts=True)[:2]
    np.testing.assert_allclose(y2, y, rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(w2, w)
    # eps does matter when it is not 0
    x3 = dict(tiny, norm_eps=1.0)
    assert not np.allclose(run(x3), y, rtol=1e-6)


def test_rmsnorm_definition_on_constant_vector():
    # RMS of a constant vector is |c|: rmsnorm(c 1, gamma, 0) = sign(c) gamma
    g = np.array([0.5, 2.0, -1.0])
    np.testing.assert_allclose(M.rmsnorm(np.full(3, -4.0), g, 0.0), -g, rtol=1e-15)
    # with eps: mean(v^2) = 16, eps = 9 -> divide by 5
    np.testing.assert_allclose(M.rmsnorm(np.full(3, 4.0), g, 9.0), 4.0 / 5.0 * g, rtol=1e-15)


def test_rope_is_the_pairwise_rotation(tiny):
    d = tiny["dims"]
    f = M._F64Inputs(tiny)
    L, half = d.kv_lora_rank, d.qk_rope_head_dim // 2
    # identity tables leave the rope part unrotated
    fi = M._F64Inputs(dict(tiny, cos=np.ones_like(tiny["cos"]), sin=np.zeros_like(tiny["sin"])))
    r0 = M.kv_row(fi, 0)[L:]
    r = M.kv_row(f, 0)[L:]
    np.testing.assert_allclose(M.kv_row(fi, 0)[:L], M.kv_row(f, 0)[:L], rtol=1e-15)
    # rotated = R(theta_i) applied to each adjacent pair of the unrotated part
    c, s = tiny["cos"][0].astype(float), tiny["sin"][0].astype(float)
    for i in range(half):
        rot = np.array([[c[i], -s[i]], [s[i], c[i]]])
        np.testing.assert_allclose(r[2 * i:2 * i + 2], rot @ r0[2 * i:2 * i + 2], rtol=1e-13, atol=1e-15)
    # a quarter turn maps (a, b) to (-b, a)
    v = np.array([3.0, 5.0, -1.0, 2.0])
    np.testing.assert_allclose(M.rope_interleaved(v, np.zeros(2), np.ones(2)), [-5.0, 3.0, -2.0, -1.0])


def test_rope_relative_position(tiny):
    # q_pe(pos) . k_pe(pos) of one token is independent of pos when the same
    # tables rotate both (the score's rope part sees only relative position).
    d = tiny["dims"]
    L = d.kv_lora_rank
    dots, scale = [], []
    for shift in (0, 17, 1000):
        c, s = synth.rope_tables(tiny["positions"] + shift, d.qk_rope_head_dim)
        f = M._F64Inputs(dict(tiny, cos=c, sin=s))
        _, q_pe = M.query_heads(f, 1)
        k_pe = M.kv_row(f, 1)[L:]
        dots.append(q_pe @ k_pe)
        scale.append(np.linalg.norm(q_pe, axis=1) * np.linalg.norm(k_pe))
    # exact in real arithmetic; the fp32-stored tables perturb it by ~1e-7
    np.testing.assert_allclose(dots[1], dots[0], rtol=0, atol=1e-6 * scale[0].max())
    np.testing.assert_allclose(dots[2], dots[0], rtol=0, atol=1e-6 * scale[0].max())


# ---------------------------------------------------------------------------
# head linearity ("this rank's" partial output)
# ---------------------------------------------------------------------------

def test_head_linearity(tiny):
    d = tiny["dims"]
    y = run(tiny)
    w = d.qk_nope_head_dim + d.qk_rope_head_dim
    total = np.zeros_like(y)
    for hs in (np.array([0, 2]), np.array([1, 3])):
        x = dict(tiny)
        x["dims"] = synth.Dims(**{**d.__dict__, "n_heads": hs.size})
        cols = np.concatenate([np.arange(h * w, (h + 1) * w) for h in hs])
        x["wq_b"] = np.ascontiguousarray(tiny["wq_b"][:, cols])
        x["q_absorb_w"] = np.ascontiguousarray(tiny["q_absorb_w"][hs])
        x["out_absorb_w"] = np.ascontiguousarray(tiny["out_absorb_w"][hs])
        rows = np.concatenate([np.arange(h * d.v_head_dim, (h + 1) * d.v_head_dim) for h in hs])
        x["o_proj_w"] = np.ascontiguousarray(tiny["o_proj_w"][rows])
        x["n_heads"] = hs.size
        total += run(x)
    np.testing.assert_allclose(total, y, rtol=1e-12, atol=1e-13 * np.abs(y).max())


# ---------------------------------------------------------------------------
# the pins catch planted mistakes
# ---------------------------------------------------------------------------

def _suite(tiny):
    check_hand_case()
    test_absorbed_equals_unabsorbed_sdpa(tiny)
    test_full_prefix_equals_dense_attention(tiny)
    test_head_linearity(tiny)
    test_rope_is_the_pairwise_rotation(tiny)


def _mutants():
    def rope_sign(v, c, s):
        a, b = v[..., 0::2], v[..., 1::2]
        out = np.empty_like(v)
        out[..., 0::2] = a * c + b * s
        out[..., 1::2] = -a * s + b * c
        return out

    def rope_halves(v, c, s):   # rotate (i, i + dr/2) instead of adjacent pairs
        h = v.shape[-1] // 2
        a, b = v[..., :h], v[..., h:]
        return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)

    def rms_eps_outside(v, g, eps):
        return v / (np.sqrt(np.mean(v * v, axis=-1, keepdims=True)) + eps) * g

    def rms_no_gamma(v, g, eps):
        return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)

    def mask_strict(bt, position, p, bs):
        if p < 0 or p >= position:
            return -1
        return int(bt[p // bs]) * bs + p % bs

    def page_swapped(bt, position, p, bs):
        if p < 0 or p > position:
            return -1
        return int(bt[p % len(bt)]) * bs + p // len(bt) % bs

    def value_with_rope(f, rows, q_lat, q_pe):
        d = f.d
        L = d.kv_lora_rank
        if rows.shape[0] == 0:
            return np.zeros((d.n_heads, d.v_head_dim))
        s = f.scale * (q_lat @ rows[:, :L].T + q_pe @ rows[:, L:].T)
        ctx = M.softmax(s) @ rows[:, :L] + (M.softmax(s) @ rows[:, L:]).sum(-1, keepdims=True)
        return np.einsum("hvl,hl->hv", f.out_absorb, ctx)

    def no_scale(f, rows, q_lat, q_pe):
        f2 = copy.copy(f)
        f2.scale = 1.0
        return orig_attend(f2, rows, q_lat, q_pe)

    def absorb_transposed(f, q_nope):
        return np.einsum("hd,hdl->hl", q_nope[:, ::-1], f.q_absorb)

    orig_attend = M.attend_token
    return [("rope_interleaved", rope_sign), ("rope_interleaved", rope_halves),
            ("rmsnorm", rms_eps_outside), ("rmsnorm", rms_no_gamma),
            ("resolve_row", mask_strict), ("resolve_row", page_swapped),
            ("attend_token", value_with_rope), ("attend_token", no_scale),
            ("absorb_query", absorb_transposed)]


@pytest.mark.parametrize("i", range(9))
def test_planted_mistakes_are_caught(tiny, monkeypatch, i):
    name, fn = _mutants()[i]
    monkeypatch.setattr(M, name, fn)
    with pytest.raises((AssertionError, ValueError, IndexError)):
        _suite(tiny)
