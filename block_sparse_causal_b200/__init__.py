"""Chunk-causal block-sparse attention over a rolling KV window, for B200 (sm_100a).

The library is ``libuf.so`` (C ABI in include/uf.h); this package binds it
with ctypes and adds a small owner of the window's device buffers.  Every step
of the hot path runs in the CUDA kernels.
"""
from ._uf import (UF_APPEND_ANCHOR, UF_APPEND_REPLACE_NEWEST, UF_EBOUNDS, UF_ECUDA, UF_EINVAL, UF_ETIMEOUT,
                  UF_EUNSUPPORTED, UF_MASK_LOCAL_ONLY, UF_OK, UfError, UfKvCache, strerror, uf_block_mask,
                  uf_attn_workspace_bytes, uf_block_mask_local, uf_block_sparse_attn, uf_block_sparse_attn_balanced,
                  uf_block_sparse_attn_balanced_noalloc,
                  uf_block_sparse_attn_fp8k, uf_check_error,
                  uf_debug_wait_timeout, uf_get_error, uf_kv_append, uf_kv_append_fp8k, uf_kv_append_rope,
                  uf_kv_append_tiled, uf_kv_cache_bytes, uf_kv_cache_init, uf_kv_cache_set_error_word, uf_kv_reset,
                  uf_rope, uf_set_clock_counters, uf_set_wait_limit, uf_source_hash, uf_tile_tokens, uf_version)
from .pipeline import ChunkPipeline
from .window import KVWindow

__all__ = [
    "UF_APPEND_ANCHOR", "UF_APPEND_REPLACE_NEWEST", "UF_EBOUNDS", "UF_ECUDA", "UF_EINVAL", "UF_ETIMEOUT",
    "UF_EUNSUPPORTED", "UF_MASK_LOCAL_ONLY", "UF_OK", "UfError", "UfKvCache", "strerror", "uf_block_mask",
    "uf_attn_workspace_bytes", "uf_block_mask_local", "uf_block_sparse_attn", "uf_block_sparse_attn_balanced",
    "uf_block_sparse_attn_balanced_noalloc",
    "uf_block_sparse_attn_fp8k", "uf_check_error",
    "uf_debug_wait_timeout", "uf_get_error", "uf_kv_append", "uf_kv_append_fp8k", "uf_kv_append_rope",
    "uf_kv_append_tiled", "uf_kv_cache_bytes", "uf_kv_cache_init", "uf_kv_cache_set_error_word", "uf_kv_reset",
    "uf_rope", "uf_set_clock_counters", "uf_set_wait_limit", "uf_source_hash", "uf_tile_tokens", "uf_version", "KVWindow", "ChunkPipeline",
]
