"""Seeded synthetic decode batches shared by the oracle tests, the CUDA parity tests
and the benchmark.

This package only builds inputs: it holds none of the attention arithmetic and
imports neither the CUDA binding nor the oracle.
"""
from .decode_batches import (  # noqa: F401
    CONFIGS,
    CONFIG_ORDER,
    DecodeBatch,
    make_batch,
    make_custom,
    permute_pool,
    unshare_prefix,
    kv_bytes,
    unique_kv_bytes,
    BF16_NAN_BITS,
    E4M3_NAN_CODE,
    fp8_scales,
    kv_element_bytes,
    PrefillBatch,
    make_prefill,
    prefill_flops,
)
