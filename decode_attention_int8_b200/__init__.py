"""q8-KV single-query decode attention for NVIDIA B200 (sm_100a).

The computation lives in libq8kv.so (CUDA kernels behind the C ABI of include/q8kv.h);
this package is its ctypes binding plus the seeded synthetic workload generators.
"""
from ._lib import (  # noqa: F401
    DEVERR_BLOCK_TABLE,
    DEVERR_META,
    DEVERR_NONFINITE,
    DEVERR_SEQ_LEN,
    DEVERR_SLOT,
    DEVERR_TIMEOUT,
    EXPORTS,
    Q8KVError,
    lib,
    lib_path,
    q8kv_cache_write,
    q8kv_cache_write_q4,
    q8kv_debug_block_dots,
    q8kv_debug_quantize_q,
    q8kv_debug_stall_pipeline,
    q8kv_decode_attn,
    q8kv_decode_attn_multi,
    q8kv_decode_attn_q4,
    q8kv_decode_attn_static,
    q8kv_decode_attn_ws,
    q8kv_quest_metadata,
    q8kv_device_errors,
    q8kv_version,
    q8kv_workspace_bytes,
    q8kv_workspace_init,
)
from . import inputs  # noqa: F401
