"""Structure of the seeded synthetic workloads (no method arithmetic involved)."""
import numpy as np
import pytest

from sparse_mla_decode_front_b200 import synth


@pytest.mark.parametrize("index", range(5))
def test_index_structure(index):
    _, d, ctx, pos, bt, gi, slot = synth.make_indices(index)
    T, P, bs = d.n_tokens, d.n_prior, d.block_size
    assert gi.shape == (T, P) and gi.dtype == np.int32
    assert bt.shape == (T, d.max_blocks_per_seq) and bt.dtype == np.int32
    assert ((bt >= 0) & (bt < d.n_blocks)).all()              # every entry a real block
    assert np.array_equal(pos, ctx - 1)
    assert len(set(slot.tolist())) == T                        # distinct slot rows
    assert (gi >= 0).all() and (gi // bs < d.max_blocks_per_seq).all()
    for t in range(T):
        assert np.unique(gi[t]).size == P                      # duplicate-free
        assert not np.all(np.diff(gi[t]) > 0)                  # unsorted
        assert int(bt[t, pos[t] // bs]) * bs + pos[t] % bs == slot[t]
    valid = gi <= pos[:, None]
    if index == 0:
        assert (valid.sum(1) == P - 4).all() and (gi <= 127).all()
        assert sorted(np.concatenate([bt[0], bt[1]]).tolist()) == list(range(16))
    elif index in (1, 2, 3):
        assert valid.all()
    elif index == 4:
        short = ctx < P
        assert (valid.sum(1)[short] == ctx[short]).all()
        assert (valid.sum(1)[~short] == P - P // 4).all()
        assert (gi <= pos[:, None] + P).all()
        for t in range(0, T - 1, 2):
            a, b = slot[t], slot[t + 1]
            assert a // bs == b // bs and a % bs != b % bs     # shared block, distinct offsets
    if index == 2:
        used = [bt[t, :(ctx[t] + bs - 1) // bs] for t in range(T)]
        allb = np.concatenate(used)
        assert np.unique(allb).size == allb.size               # disjoint across sequences
    if index == 3:
        cur = bt[np.arange(T), pos // bs]
        assert np.unique(cur).size == T
        others = np.delete(bt.reshape(-1), np.arange(T) * d.max_blocks_per_seq + pos // bs)
        assert not np.isin(cur, others).any()                  # current blocks exclusive
        assert np.unique(others).size < others.size            # others shared


def test_seeded_and_deterministic():
    a = synth.make_inputs(0)
    b = synth.make_inputs(0)
    for k in synth.TENSOR_ARGS:
        assert np.array_equal(a[k], b[k]), k
    c = synth.make_inputs(0, seed=77)
    assert not np.array_equal(a["hidden_states"], c["hidden_states"])


def test_value_distributions():
    x = synth.make_inputs(0)
    d = x["dims"]
    w = synth.bf16_bits_to_f32(x["wq_b"]).astype(np.float64)
    assert abs(w.std() * np.sqrt(d.q_lora_rank) - 1) < 0.05
    g = x["input_norm_w"].astype(np.float64)
    assert abs(g.mean() - 1) < 0.03 and abs(g.std() - 0.1) < 0.03
    flat = x["kv_cache"].reshape(-1, d.kv_row_dim)
    filled = synth.bf16_bits_to_f32(flat[x["cache_fill_rows"]])
    assert abs(filled.std() - 1) < 0.05
    c, s = x["cos"], x["sin"]
    np.testing.assert_allclose(c * c + s * s, 1.0, atol=1e-6)
    np.testing.assert_allclose(c[:, 0], np.cos(x["positions"].astype(np.float64)), atol=1e-7)


def test_bf16_sample_rounding_matches_torch():
    import torch
    v = np.random.default_rng(1).standard_normal(10000).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(synth.f32_to_bf16_bits(v), ref)
