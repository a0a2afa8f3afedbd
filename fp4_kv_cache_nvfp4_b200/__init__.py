"""CSA2 sparse global attention over an NVFP4 main-KV cache, for B200 (sm_100a).

Thin Python binding of the C ABI in ``include/csa2.h`` (library
``libcsa2.so``, built in-tree by ``fp4_kv_cache_nvfp4_b200.build``).  The
binding only marshals arguments: every step of the path runs in the library's
CUDA kernels.  PyTorch provides device memory and streams.  There is no CPU
fallback: without the built library, importing the binding raises.
"""
from __future__ import annotations

import ctypes
import os

from ._binding import (  # noqa: F401
    BLOCK, BF16, CSA2Error, F32, FULL, KVCache, LayerDesc, REINDEX, REUSE, TOKEN, abi_version, attn_lse_merge,
    decode_layers, default_desc, device_accessible, indexer_score_ids, indexer_topk, indexer_topk_noalloc,
    kv_quant_append, lib, lib_path, schedule, sparse_attn_decode, sparse_attn_prefill, swa_replay, test_empty_chain,
    test_set_wait_limit, topk_merge, workspace_bytes,
)
