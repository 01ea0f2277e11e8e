"""CPU fp64 oracle of the fused RMSNorm + router top-K step of a MoE decoder layer.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
execute this module; only ``tests/`` and the measurement legs of ``bench.py``
use it. It shares no code, tables or constants with the CUDA path.

What it computes follows the page "RMSNorm Router Top-K A2AV Kernel API
Reference" (AWS Neuron NKI library, ``rmsnorm_router_topk_a2av``), section
"API Reference" (:param and :return entries) and its "Notes". The page prints no
equations; each step restates an entry, and where the page is open the plainest
reading is taken and named here:

* norm = x / sqrt(mean(x^2) + eps) * gamma per token (:param hidden_states,
  gamma, eps), the first output, stored in the input's dtype (bf16: rounded once
  to nearest-even).
* logits = norm @ router_weights (+ router_bias) (:param router_weights,
  router_bias). Reading: the router consumes the normalised states as computed,
  before their bf16 store; the bias is added to every logit.
* The top-K experts are chosen on these raw logits, before any activation
  (Notes: "top-K on raw logits, then activation applied only to selected
  experts"). Reading: largest logit first; equal logits are taken in increasing
  expert index; the K indices are listed in that order.
* Affinities (:return [T, E] masked affinities): the activation of the selected
  experts' logits, zero for every other expert. SIGMOID: sigmoid(logit) per
  selected expert. SOFTMAX: reading: a softmax over the K selected logits only
  (the activation is applied to the selected experts alone).

Precision: inputs are read exactly from their bf16 storage and every operation
is fp64; the only roundings are the two stores the page fixes as bf16 (norm and
affinities).

Pins (tests/test_router_pins.py) tie these functions to facts fixed outside
this file: brute force over every K-subset on tiny inputs, one-hot router
columns, RMSNorm scale invariance, activation closed forms, bias dominance and
expert-permutation equivariance.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from .mla_block import bf16_to_f64, f64_to_bf16

SIGMOID = "sigmoid"
SOFTMAX = "softmax"


def normalize(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm of each token row: x / sqrt(mean(x^2) + eps) * gamma (fp64)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gamma


def router_logits(norm: np.ndarray, weights: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    """Raw router logits [T, E] = norm [T, H] @ router_weights [H, E] (+ bias [E])."""
    logits = norm @ weights
    if bias is not None:
        logits = logits + bias
    return logits


def topk_desc(logits: np.ndarray, k: int) -> np.ndarray:
    """Per row, the k largest logits' expert indices, largest first, equal logits in
    increasing index (int32 [T, k])."""
    E = logits.shape[-1]
    order = np.lexsort((np.broadcast_to(np.arange(E), logits.shape), -logits), axis=-1)
    return order[..., :k].astype(np.int32)


def activate(logits: np.ndarray, idx: np.ndarray, act: str) -> np.ndarray:
    """Masked affinities [T, E]: the activation of the selected logits, 0 elsewhere."""
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=-1)
    if act == SIGMOID:
        a = 1.0 / (1.0 + np.exp(-sel))
    elif act == SOFTMAX:
        e = np.exp(sel - sel.max(axis=-1, keepdims=True))
        a = e / e.sum(axis=-1, keepdims=True)
    else:
        raise ValueError(f"unknown router activation {act!r}")
    out = np.zeros_like(logits)
    np.put_along_axis(out, idx.astype(np.int64), a, axis=-1)
    return out


def rmsnorm_router_topk(inp: Dict[str, object]) -> Dict[str, np.ndarray]:
    """The step on one input set (bf16 bit patterns as uint16; see synth.make_router_inputs).

    Returns fp64 ``norm``, ``logits`` and ``affinities``, their bf16 stores
    ``norm_bits`` / ``aff_bits``, and ``idx`` [T, K] int32."""
    x = bf16_to_f64(inp["hidden_states"])
    gamma = bf16_to_f64(inp["gamma"])
    w = bf16_to_f64(inp["router_weights"])
    bias = None if inp.get("router_bias") is None else bf16_to_f64(inp["router_bias"])
    norm = normalize(x, gamma, float(inp["eps"]))
    logits = router_logits(norm, w, bias)
    idx = topk_desc(logits, int(inp["top_k"]))
    aff = activate(logits, idx, str(inp["act"]))
    return dict(norm=norm, norm_bits=f64_to_bf16(norm), logits=logits, idx=idx, affinities=aff,
                aff_bits=f64_to_bf16(aff))
