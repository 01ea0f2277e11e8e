"""Pins of the fused RMSNorm + router top-K oracle (oracle/router_topk.py) to facts
fixed outside it (page "RMSNorm Router Top-K A2AV Kernel API Reference": :param
hidden_states, gamma, router_weights, router_bias, eps, top_k, router_act_fn;
:return entries; Notes on the top-K / activation order).
"""
import itertools
import math

import numpy as np
import pytest

from oracle import router_topk as R
from oracle.mla_block import bf16_to_f64
from sparse_mla_decode_front_b200 import synth

bf = lambda v: synth.f32_to_bf16_bits(np.asarray(v, np.float32))


def _inp(x, gamma, w, bias=None, k=1, act="sigmoid", eps=1e-6):
    return dict(hidden_states=bf(x), gamma=bf(gamma), router_weights=bf(w),
                router_bias=None if bias is None else bf(bias), eps=eps, top_k=k, act=act)


def test_hand_case():
    # T=1, H=2, E=3, K=2, gamma = 1, eps = 0: x = (3, 4), mean(x^2) = 12.5, so
    # norm = x / sqrt(12.5) = (0.8485281374, 1.1313708499). Router columns
    # (1, 0), (0, 1), (1, -1) give logits (0.8485..., 1.1313..., -0.2828...):
    # expert 1 then expert 0.
    w = [[1.0, 0.0, 1.0], [0.0, 1.0, -1.0]]
    s = 1.0 / math.sqrt(12.5)
    norm = (3 * s, 4 * s)
    logits = (norm[0], norm[1], norm[0] - norm[1])
    for act in ("sigmoid", "softmax"):
        o = R.rmsnorm_router_topk(_inp([[3.0, 4.0]], [1.0, 1.0], w, k=2, act=act, eps=0.0))
        np.testing.assert_allclose(o["norm"][0], norm, rtol=1e-15)
        np.testing.assert_allclose(o["logits"][0], logits, rtol=1e-14)
        assert o["idx"].tolist() == [[1, 0]]
        if act == "sigmoid":
            want = (1 / (1 + math.exp(-logits[0])), 1 / (1 + math.exp(-logits[1])), 0.0)
        else:   # softmax over the two selected logits only
            d = math.exp(logits[1] - logits[0])
            want = (1 / (1 + d), d / (1 + d), 0.0)
        np.testing.assert_allclose(o["affinities"][0], want, rtol=1e-14)
    # numbers worked by hand: sigmoid(0.84853) = 0.70026, sigmoid(1.13137) = 0.75610
    o = R.rmsnorm_router_topk(_inp([[3.0, 4.0]], [1.0, 1.0], w, k=2, eps=0.0))
    np.testing.assert_allclose(o["affinities"][0, :2], (0.70026, 0.75610), atol=1e-5)


def test_brute_force_topk_over_all_subsets():
    # Tiny case: logits by explicit loops, the top-K set as the K-subset with the
    # largest logit sum (unique here) found by enumerating every subset.
    inp = synth.make_router_inputs(0)
    c = inp["case"]
    o = R.rmsnorm_router_topk(inp)
    x = bf16_to_f64(inp["hidden_states"])
    g = bf16_to_f64(inp["gamma"])
    w = bf16_to_f64(inp["router_weights"])
    b = bf16_to_f64(inp["router_bias"])
    for t in range(c.n_tokens):
        ss = 0.0
        for h in range(c.hidden):
            ss += x[t, h] * x[t, h]
        r = 1.0 / math.sqrt(ss / c.hidden + inp["eps"])
        lg = []
        for e in range(c.n_experts):
            acc = 0.0
            for h in range(c.hidden):
                acc += x[t, h] * r * g[h] * w[h, e]
            lg.append(acc + b[e])
        np.testing.assert_allclose(o["logits"][t], lg, rtol=1e-12, atol=1e-12)
        best = max(itertools.combinations(range(c.n_experts), c.top_k), key=lambda s: sum(lg[e] for e in s))
        assert set(o["idx"][t].tolist()) == set(best)
        vals = [lg[e] for e in o["idx"][t]]
        assert vals == sorted(vals, reverse=True)   # listed largest first
        assert np.count_nonzero(o["affinities"][t]) == c.top_k
        np.testing.assert_allclose(o["affinities"][t].sum(), 1.0, rtol=1e-12)   # softmax over the selected


def test_one_hot_router_columns_read_the_normalised_states():
    # Column e of the router picks hidden position p_e: logit = norm[t, p_e].
    rng = np.random.default_rng(7)
    T, H, E = 4, 64, 8
    x = rng.standard_normal((T, H))
    gamma = 1.0 + 0.1 * rng.standard_normal(H)
    pos = rng.permutation(H)[:E]
    w = np.zeros((H, E))
    w[pos, np.arange(E)] = 1.0
    inp = _inp(x, gamma, w, k=3)
    o = R.rmsnorm_router_topk(inp)
    xb, gb = bf16_to_f64(inp["hidden_states"]), bf16_to_f64(inp["gamma"])
    norm = xb / np.sqrt((xb ** 2).mean(axis=1, keepdims=True) + 1e-6) * gb
    np.testing.assert_allclose(o["logits"], norm[:, pos], rtol=1e-14)
    for t in range(T):
        assert set(o["idx"][t]) == set(np.argsort(-norm[t, pos])[:3])


def test_rmsnorm_scale_invariance():
    inp = synth.make_router_inputs(3)
    inp["eps"] = 0.0
    o1 = R.rmsnorm_router_topk(inp)
    scaled = dict(inp)
    scaled["hidden_states"] = synth.f32_to_bf16_bits(4.0 * synth.bf16_bits_to_f32(inp["hidden_states"]))
    o2 = R.rmsnorm_router_topk(scaled)
    np.testing.assert_allclose(o2["norm"], o1["norm"], rtol=1e-14)
    np.testing.assert_array_equal(o2["idx"], o1["idx"])


@pytest.mark.parametrize("act,want", [("sigmoid", 0.5), ("softmax", 0.25)])
def test_equal_logits_take_the_lowest_indices(act, want):
    # Zero router and no bias: every logit is 0, so the ties take experts 0..K-1 and the
    # activation gives sigmoid(0) = 1/2, or a uniform 1/K softmax.
    inp = _inp(np.ones((2, 32)), np.ones(32), np.zeros((32, 10)), k=4, act=act)
    o = R.rmsnorm_router_topk(inp)
    assert o["idx"].tolist() == [[0, 1, 2, 3]] * 2
    np.testing.assert_allclose(o["affinities"][:, :4], want, rtol=1e-15)
    assert not o["affinities"][:, 4:].any()


def test_bias_dominates_the_selection():
    inp = synth.make_router_inputs(3)
    c = inp["case"]
    bias = bf16_to_f64(inp["router_bias"]).copy()
    bias[17], bias[40] = 100.0, -100.0
    inp["router_bias"] = bf(bias)
    o = R.rmsnorm_router_topk(inp)
    assert (o["idx"][:, 0] == 17).all()
    assert not (o["idx"] == 40).any()
    assert o["idx"].shape == (c.n_tokens, c.top_k)


def test_expert_permutation_equivariance():
    inp = synth.make_router_inputs(3)
    o = R.rmsnorm_router_topk(inp)
    perm = np.random.default_rng(3).permutation(inp["case"].n_experts)
    p = dict(inp)
    p["router_weights"] = inp["router_weights"][:, perm]
    p["router_bias"] = inp["router_bias"][perm]
    op = R.rmsnorm_router_topk(p)
    np.testing.assert_array_equal(op["logits"], o["logits"][:, perm])
    for t in range(inp["case"].n_tokens):
        assert set(perm[op["idx"][t]]) == set(o["idx"][t])
    np.testing.assert_array_equal(op["affinities"], o["affinities"][:, perm])


def test_stored_outputs_are_one_rounding():
    # each stored value (norm, affinities) is within half a bf16 spacing of the fp64 value
    o = R.rmsnorm_router_topk(synth.make_router_inputs(0))
    for key, bits in (("norm", "norm_bits"), ("affinities", "aff_bits")):
        v, s = o[key], bf16_to_f64(o[bits])
        _, e = np.frexp(np.where(v == 0, 1.0, v))
        assert (np.abs(s - v) <= np.ldexp(1.0, e - 9) + 1e-300).all()
