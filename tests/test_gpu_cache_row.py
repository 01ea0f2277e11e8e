"""The cache row on inputs built to stress its one-ulp bar (page "MLA Attention
Block Gather Decode Kernel API Reference", :param kv_cache: the front-fold
writes this step's bf16 row).

The CUDA path rounds each row element once from an fp32 value whose error is
fp32 accumulation of the KV down-projection, and recomputes in fp64 the
elements smaller than 2^-8 of the row's RMS (latent part; per rotated pair for
the rope part). These tests aim at that split:

  * a hidden row with a large dynamic range (elements spread over 2^-16 .. 2^8),
    so the dot products cancel heavily and the fp32 error is largest relative to
    the result;
  * latent elements placed just below and just above the recompute threshold
    (0.9 .. 1.1 of it), on both sides and both signs, by adjusting single weight
    entries until the exact pre-norm value hits its target.

Both compare every written row, element by element, with the oracle's row (the
fp64 row rounded once), and require at most one bf16 ulp.
"""
import numpy as np
import pytest

import oracle
from sparse_mla_decode_front_b200 import synth
from test_gpu_parity import ROW_ULPS, gpu_run, ulp_distance

pytestmark = pytest.mark.gpu

TAU = 2.0 ** -8   # the recompute threshold, relative to the latent RMS


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _f(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _rows_only(inp):
    x = dict(inp)
    x["kv_cache"] = inp["kv_cache"].copy()
    _, written, _ = oracle.block(x, tokens=[], return_parts=True)
    return written


def _check_rows(inp):
    _, rows_gpu, status, _ = gpu_run(inp)
    assert status == 0, f"device status {status:#x}"
    rows_ref = _rows_only(inp)
    ulps = ulp_distance(rows_gpu, rows_ref)
    assert ulps.max() <= ROW_ULPS, f"{(ulps > ROW_ULPS).sum()} elements beyond {ROW_ULPS} ulp"
    return ulps


def test_large_dynamic_range_hidden():
    inp = dict(synth.make_inputs(2))   # 32 tokens, DeepSeek-V3.2 dims
    rng = np.random.default_rng(91)
    d = inp["dims"]
    scale = 2.0 ** rng.uniform(-16, 8, size=(d.n_tokens, d.hidden))
    inp["hidden_states"] = _bf16(rng.standard_normal((d.n_tokens, d.hidden)) * scale)
    _check_rows(inp)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_latent_elements_at_the_recompute_threshold(seed):
    # One token (the weight column a target adjusts is shared by every token, so each
    # case targets one row), 24 latent elements at 0.9 .. 1.1 of the threshold.
    inp = dict(synth.make_inputs(1, seed=None if seed == 0 else 5000 + seed))
    d = inp["dims"]
    L, R = d.kv_lora_rank, d.kv_row_dim
    x = _f(inp["hidden_states"])                                 # [T, H]
    g = np.asarray(inp["input_norm_w"], dtype=np.float32)
    xg = (x.astype(np.float32) * g).astype(np.float64)           # the fp32 product the path splits exactly
    w_bits = inp["wkv_a"].copy().reshape(d.hidden, R)
    w = _f(w_bits)
    factors = [0.9, 0.99, 0.999, 0.9999, 1.0001, 1.001, 1.01, 1.1, -0.995, -0.9999, -1.0001, -1.005] * 2
    targets = [(0, [17 * i + seed for i in range(len(factors))])]   # spread over the latent columns
    mag = np.abs(xg)
    for _ in range(3):   # the RMS moves a little as the targeted columns move
        kv = xg @ w
        rms = np.sqrt(np.mean(kv[:, :L] ** 2, axis=1))
        for t, cols in targets:
            for c, f in zip(cols, factors):
                want = f * TAU * rms[t]
                used = set()
                for _ in range(5):
                    # one weight entry takes the residual; its x*gamma is chosen so that the new
                    # weight is about 0.05, which its bf16 rounding then resolves to 2^-9 of the
                    # residual, so each step shrinks the residual by about 2^9
                    delta = want - xg[t] @ w[:, c]
                    if delta == 0.0:
                        break
                    dist = np.abs(mag[t] - abs(delta) / 0.05)
                    dist[list(used)] = np.inf
                    dist[mag[t] == 0.0] = np.inf
                    k = int(np.argmin(dist))
                    used.add(k)
                    w_bits[k, c] = _bf16(np.float64(w[k, c] + delta / xg[t, k])).item()
                    w[k, c] = float(_f(np.asarray(w_bits[k, c])))
    kv = xg @ w
    rms = np.sqrt(np.mean(kv[:, :L] ** 2, axis=1))
    rel = np.array([[kv[t, c] / (TAU * rms[t]) for c in cols] for t, cols in targets])
    assert np.abs(rel - np.array(factors)).max() < 2e-5, "targets not reached"
    inp["wkv_a"] = w_bits.reshape(inp["wkv_a"].shape)
    _check_rows(inp)
