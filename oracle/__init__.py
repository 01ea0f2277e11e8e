"""CPU fp64 oracle of the sparse MLA gather-decode block.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline / reference legs of bench.py. The product path never imports it.
"""
from .mla_block import (bf16_to_f64, f64_to_bf16, rmsnorm, rope_interleaved, resolve_row,
                        softmax, kv_row, query_heads, absorb_query, attend_token, o_projection,
                        head_split_output, block)

__all__ = ["bf16_to_f64", "f64_to_bf16", "rmsnorm", "rope_interleaved", "resolve_row",
           "softmax", "kv_row", "query_heads", "absorb_query", "attend_token", "o_projection",
           "head_split_output", "block"]
