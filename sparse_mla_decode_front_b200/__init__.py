"""B200 (sm_100a) sparse MLA gather-decode block.

One DeepSeek-V3.2 MLA decode step from the residual stream to the attention-
block output, attending only over indexer-selected prior keys, as defined by
the page "MLA Attention Block Gather Decode Kernel API Reference". The work
runs in hand-written CUDA kernels behind a C ABI (include/sparse_mla_decode.h);
this package binds it (``api``), keeps a step's tensors resident (``device``)
and generates seeded synthetic workloads (``synth``).
"""
from .api import (mla_abi_version, mla_attention_block_gather_decode, mla_block_check_dims,
                  mla_block_gather_decode, mla_block_workspace_bytes, mla_get_device_status,
                  mla_status_string)
from ._lib import MlaError

__all__ = ["mla_abi_version", "mla_attention_block_gather_decode", "mla_block_check_dims",
           "mla_block_gather_decode", "mla_block_workspace_bytes", "mla_get_device_status",
           "mla_status_string", "MlaError"]
