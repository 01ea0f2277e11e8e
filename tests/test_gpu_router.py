"""The fused RMSNorm + router top-K on the GPU against the fp64 oracle
(oracle/router_topk.py; page "RMSNorm Router Top-K A2AV Kernel API Reference").

Bars: the norm row within 1 bf16 ulp of the oracle's rounded row; the selected
experts are a valid top-K of the oracle's logits (equal to the oracle's set
wherever its K-th and (K+1)-th logits are further apart than the logits' fp32
accumulation error), listed largest first; the affinities of the selected experts
within bf16 rounding of the activation of those experts' oracle logits, and
exactly 0 elsewhere.
"""
import numpy as np
import pytest
import torch

from oracle import router_topk as R
from oracle.mla_block import bf16_to_f64
from sparse_mla_decode_front_b200 import api, synth
from test_gpu_parity import ulp_distance

pytestmark = pytest.mark.gpu

LOGIT_TOL = 1e-4   # relative to max(1, max |logit|): far above fp32 accumulation over H terms


def bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run_gpu(inp, shape=None):
    x = bf16_tensor(inp["hidden_states"])
    if shape is not None:
        x = x.reshape(shape)
    b = None if inp["router_bias"] is None else bf16_tensor(inp["router_bias"])
    norm, idx, aff = api.rmsnorm_router_topk(x, bf16_tensor(inp["gamma"]), bf16_tensor(inp["router_weights"]), b,
                                             inp["eps"], inp["top_k"], inp["act"])
    torch.cuda.synchronize()
    as_bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    return as_bits(norm), idx.cpu().numpy(), bf16_to_f64(as_bits(aff))


def check(inp, norm_bits, idx, aff):
    ref = R.rmsnorm_router_topk(inp)
    K, E = int(inp["top_k"]), ref["logits"].shape[1]
    assert ulp_distance(norm_bits, ref["norm_bits"]).max() <= 1
    L = ref["logits"]
    for t in range(L.shape[0]):
        tol = LOGIT_TOL * max(1.0, np.abs(L[t]).max())
        sel = idx[t]
        assert len(set(sel.tolist())) == K and sel.min() >= 0 and sel.max() < E
        srt = np.sort(L[t])[::-1]
        assert L[t, sel].min() >= srt[K - 1] - tol                      # a valid top-K
        if K < E and srt[K - 1] - srt[K] > tol:
            assert set(sel.tolist()) == set(ref["idx"][t].tolist())     # unique here
        assert (np.diff(L[t, sel]) <= tol).all()                        # largest first
        want = R.activate(L[t:t + 1], sel[None].astype(np.int32), inp["act"])[0]
        mask = np.zeros(E, bool)
        mask[sel] = True
        assert not aff[t, ~mask].any()
        np.testing.assert_allclose(aff[t, mask], want[mask], rtol=2.0 ** -8, atol=1e-6)


@pytest.mark.parametrize("case", ["router_ds128", "router_one", "router_ragged", "router_tall", "router_wide",
                                  "router_odd"])
def test_router_matches_oracle(case):
    inp = synth.make_router_inputs(synth.ROUTER_CASE_BY_NAME[case].index)
    check(inp, *run_gpu(inp))


@pytest.mark.parametrize("case,launches", [("router_ds128", 1), ("router_one", 1), ("router_tall", 1),
                                           ("router_odd", 1), ("router_wide", 3)])
def test_router_launch_count(case, launches):
    # up to 256 experts: one cooperative launch (partial logits, grid barrier, finish);
    # wider: prep, projection and finish
    c = synth.ROUTER_CASE_BY_NAME[case]
    inp = synth.make_router_inputs(c.index)
    x = bf16_tensor(inp["hidden_states"])
    T, H, E = c.n_tokens, c.hidden, c.n_experts
    norm = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, c.top_k), dtype=torch.int32, device="cuda")
    aff = torch.empty((T, E), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(api.mla_router_workspace_bytes(T, H, E, c.top_k), dtype=torch.uint8, device="cuda")
    assert api.mla_router_launches(T, H, E, c.top_k) == launches
    api.mla_rmsnorm_router_topk(x, bf16_tensor(inp["gamma"]), bf16_tensor(inp["router_weights"]),
                                None if inp["router_bias"] is None else bf16_tensor(inp["router_bias"]), inp["eps"],
                                c.top_k, inp["act"], norm, idx, aff, ws)
    torch.cuda.synchronize()
    check(inp, norm.view(torch.int16).cpu().numpy().view(np.uint16), idx.cpu().numpy(),
          bf16_to_f64(aff.view(torch.int16).cpu().numpy().view(np.uint16)))


@pytest.mark.parametrize("act", ["sigmoid", "softmax"])
def test_router_both_activations_and_no_bias(act):
    inp = synth.make_router_inputs(synth.ROUTER_CASE_BY_NAME["router_ragged"].index)
    inp["act"], inp["router_bias"] = act, None
    check(inp, *run_gpu(inp))


def test_router_page_style_batch_shape_and_bias_dominance():
    # [B, S, H] input as the page takes it; a large bias forces one expert first.
    inp = synth.make_router_inputs(synth.ROUTER_CASE_BY_NAME["router_ds128"].index)
    bias = bf16_to_f64(inp["router_bias"]).copy()
    bias[200] = 50.0
    inp["router_bias"] = synth.f32_to_bf16_bits(bias.astype(np.float32))
    norm_bits, idx, aff = run_gpu(inp, shape=(2, 64, 7168))
    assert (idx[:, 0] == 200).all()
    check(inp, norm_bits, idx, aff)


def test_router_rejects_bad_calls_before_launch():
    inp = synth.make_router_inputs(synth.ROUTER_CASE_BY_NAME["router_one"].index)
    x = bf16_tensor(inp["hidden_states"])
    g, w = bf16_tensor(inp["gamma"]), bf16_tensor(inp["router_weights"])
    with pytest.raises(ValueError, match="activation"):
        api.rmsnorm_router_topk(x, g, w, None, 1e-6, 6, "relu")
    with pytest.raises(api.MlaError):
        api.rmsnorm_router_topk(x, g, w, None, 1e-6, 33, "sigmoid")   # top_k beyond 32
