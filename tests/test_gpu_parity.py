"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Bars (the block's stated tolerances):
  * the cache row each token writes: within 1 bf16 ulp of the oracle's row
    (the fp64 row rounded once to bf16), element by element;
  * the block output: max|gpu - oracle| / max|oracle| <= 1e-2 (bf16 I/O,
    fp32 accumulation), over the tokens compared.
Every workload is compared on every token, in the same launch configuration
the benchmark times (the oracle writes every token's row first).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_mla_decode_front_b200 import _lib, api, synth
from sparse_mla_decode_front_b200.device import DecodeStep

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
ROW_ULPS = 1


def ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Number of bf16 steps between two bf16 bit arrays (adjacent values -> 1)."""
    def key(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(key(a) - key(b))


def gpu_run(inp, repeat=1):
    step = DecodeStep(inp)
    for _ in range(repeat):
        out = step.run()
    torch.cuda.synchronize()
    d = inp["dims"]
    cache = step.t["kv_cache"].view(-1, d.kv_row_dim)
    slots = torch.from_numpy(inp["slot_mapping"].astype(np.int64)).cuda()
    rows = cache[slots].view(torch.int16).cpu().numpy().view(np.uint16)
    y = out.float().cpu().numpy().astype(np.float64)
    return y, rows, step.device_status(), step


def oracle_run(inp, tokens=None):
    x = dict(inp)
    x["kv_cache"] = inp["kv_cache"].copy()
    y, written, _ = oracle.block(x, tokens=tokens, return_parts=True)
    return y, written


def check(inp, tokens=None):
    y_gpu, rows_gpu, status, _ = gpu_run(inp)
    assert status == 0, f"device status {status:#x}"
    y_ref, rows_ref = oracle_run(inp, tokens)
    ulps = ulp_distance(rows_gpu, rows_ref)
    assert ulps.max() <= ROW_ULPS, f"cache row off by {ulps.max()} ulp at {np.argwhere(ulps > ROW_ULPS)[:5]}"
    sel = slice(None) if tokens is None else list(tokens)
    err = np.abs(y_gpu[sel] - y_ref).max() / np.abs(y_ref).max()
    assert err <= OUT_TOL, f"output rel err {err:.3e}"
    return err, ulps


@pytest.fixture(scope="module")
def tiny():
    return synth.make_inputs(0)


def test_tiny_all_tokens(tiny):
    check(tiny)


def test_slice16_all_tokens():
    check(synth.make_inputs(1))


@pytest.mark.slow
def test_batch32_all_tokens():
    check(synth.make_inputs(2))


@pytest.mark.slow
def test_gather128_all_tokens():
    check(synth.make_inputs(3))


@pytest.mark.slow
def test_mask64_all_tokens():
    # includes contexts shorter than n_prior, future (masked) entries and tokens whose
    # current rows share a physical block
    check(synth.make_inputs(4))


@pytest.mark.slow
def test_gather128_every_token_within_bar():
    # each token on its own scale: max|gpu - oracle| / max|oracle| per token row
    inp = synth.make_inputs(3)
    y_gpu, _, status, _ = gpu_run(inp)
    assert status == 0
    y_ref, _ = oracle_run(inp)
    per_tok = np.abs(y_gpu - y_ref).max(axis=1) / np.abs(y_ref).max(axis=1)
    assert per_tok.max() <= OUT_TOL, f"worst token {int(per_tok.argmax())}: {per_tok.max():.3e}"


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

def test_repeat_calls_are_idempotent(tiny):
    y1, r1, s1, _ = gpu_run(tiny, repeat=1)
    y2, r2, s2, _ = gpu_run(tiny, repeat=3)
    assert s1 == 0 and s2 == 0
    np.testing.assert_array_equal(r1, r2)
    np.testing.assert_allclose(y1, y2, rtol=0, atol=0)


def test_all_keys_masked_gives_zero(tiny):
    x = dict(tiny)
    x["gather_indices"] = np.full_like(tiny["gather_indices"], 127)
    x["gather_indices"][:, ::3] = -7
    y, rows, status, _ = gpu_run(x)
    assert status == 0
    assert np.all(y == 0.0)
    _, rows_ref = oracle_run(x)
    assert ulp_distance(rows, rows_ref).max() <= ROW_ULPS


def test_no_prior_keys(tiny):
    x = dict(tiny)
    x["gather_indices"] = np.zeros((2, 0), np.int32)
    x["dims"] = synth.Dims(**{**tiny["dims"].__dict__, "n_prior": 0})
    y, rows, status, _ = gpu_run(x)
    assert status == 0 and np.all(y == 0.0)


def test_own_row_only(tiny):
    # Each token selects only its own position: attends to the row it writes.
    x = dict(tiny)
    g = np.full_like(tiny["gather_indices"], 127)
    g[:, 5] = tiny["positions"]
    x["gather_indices"] = g
    check(x)


def test_bad_block_id_is_flagged_and_masked(tiny):
    d = tiny["dims"]
    x = dict(tiny)
    bt = tiny["block_table"].copy()
    t, p = 0, int(tiny["gather_indices"][0][np.argmax(tiny["gather_indices"][0] <= tiny["positions"][0])])
    bt[t, p // d.block_size] = d.n_blocks + 3
    x["block_table"] = bt
    y, _, status, _ = gpu_run(x)
    assert status & _lib.MLA_DEV_BAD_BLOCK_ID
    # same as the oracle with every key of that logical block masked
    ref = dict(tiny)
    g = tiny["gather_indices"].copy()
    g[t][g[t] // d.block_size == p // d.block_size] = -1
    ref["gather_indices"] = g
    y_ref, _ = oracle_run(ref)
    assert np.abs(y - y_ref).max() / np.abs(y_ref).max() <= OUT_TOL


def test_bad_slot_is_flagged(tiny):
    x = dict(tiny)
    s = tiny["slot_mapping"].copy()
    s[1] = -4
    x["slot_mapping"] = s
    _, _, status, _ = gpu_run(x)
    assert status & _lib.MLA_DEV_BAD_SLOT


def test_page_style_call_matches(tiny):
    y_ref, _, _, step = gpu_run(tiny)
    t = {k: v.clone() for k, v in step.t.items()}
    d = tiny["dims"]
    out = api.mla_attention_block_gather_decode(
        t["hidden_states"], t["input_norm_w"], t["wq_a"], t["q_norm_w"], t["wq_b"], t["wkv_a"],
        t["kv_norm_w"], t["q_absorb_w"], t["out_absorb_w"], t["o_proj_w"], t["cos"], t["sin"],
        t["kv_cache"], t["slot_mapping"], t["block_table"], t["positions"], t["gather_indices"],
        n_heads=d.n_heads, qk_nope_head_dim=d.qk_nope_head_dim, qk_rope_head_dim=d.qk_rope_head_dim,
        kv_lora_rank=d.kv_lora_rank, softmax_scale=tiny["softmax_scale"])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.float().cpu().numpy(), y_ref)


def test_side_stream_and_host_path(tiny):
    step = DecodeStep(tiny)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = step.run_from_host(s)
    s.synchronize()
    y_ref, _ = oracle_run(tiny)
    yy = y.float().numpy().astype(np.float64)
    assert np.abs(yy - y_ref).max() / np.abs(y_ref).max() <= OUT_TOL


def test_pipelined_host_steps(tiny):
    # Back-to-back steps with overlapped host copies (two device buffer sets, two copy
    # streams): every step computes the same block, so the last step's output read back
    # to the host matches the oracle, and the cache rows are the oracle's.
    y_ref, rows_ref = oracle_run(tiny)
    step = DecodeStep(tiny)
    for graphs in (False, True):
        ms = step.pipeline_from_host(5, graphs=graphs)
        torch.cuda.synchronize()
        assert ms > 0 and step.device_status() == 0
        y = step.pipe_last_out.float().numpy().astype(np.float64)
        assert np.abs(y - y_ref).max() / np.abs(y_ref).max() <= OUT_TOL
    d = tiny["dims"]
    cache = step.t["kv_cache"].view(-1, d.kv_row_dim)
    slots = torch.from_numpy(tiny["slot_mapping"].astype(np.int64)).cuda()
    rows = cache[slots].view(torch.int16).cpu().numpy().view(np.uint16)
    assert ulp_distance(rows, rows_ref).max() <= ROW_ULPS
