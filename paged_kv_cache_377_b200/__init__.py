"""Paged KV-cache decode attention for B200 (sm_100a).

A thin binding over the C ABI of ``libpagedkv.so`` (see include/pagedkv.h):
argument marshalling only -- every step of the decode path runs in the CUDA
kernels of the library. Tensors are torch tensors on the GPU; torch supplies
device memory and streams. If the library cannot be loaded (or built with
nvcc), every call raises: there is no CPU fallback.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    DecodeAppendCall,
    DecodeAppendFp8Call,
    PKV_MAX_PREFIX_GROUPS,
    PKV_STATUS_BAD_BLOCK_ID,
    PKV_STATUS_BAD_CONTEXT_LEN,
    PKV_STATUS_BAD_PREFIX_GROUP,
    PKV_STATUS_BAD_SLOT,
    PKV_STATUS_WAIT_TIMEOUT,
    PagedKVError,
    PrefixGroups,
    allocate_workspace,
    find_prefix_groups,
    kv_cache_append,
    kv_cache_append_fp8,
    library,
    library_path,
    paged_attn_decode,
    paged_attn_decode_append,
    paged_attn_decode_append_fp8,
    paged_attn_decode_fp8,
    paged_attn_decode_noalloc,
    paged_attn_prefill,
    read_status,
    selftest_bounded_wait,
    validate,
    workspace_bytes,
)
from .block_manager import BlockManager, OutOfBlocks, kv_block_copy  # noqa: F401

__all__ = [
    "BlockManager",
    "DecodeAppendCall",
    "DecodeAppendFp8Call",
    "OutOfBlocks",
    "PagedKVError",
    "PrefixGroups",
    "allocate_workspace",
    "find_prefix_groups",
    "kv_block_copy",
    "kv_cache_append",
    "library",
    "library_path",
    "paged_attn_decode",
    "paged_attn_decode_append",
    "paged_attn_decode_append_fp8",
    "paged_attn_decode_fp8",
    "paged_attn_decode_noalloc",
    "paged_attn_prefill",
    "kv_cache_append_fp8",
    "read_status",
    "validate",
    "workspace_bytes",
]
