"""paged_kv_cache_406_b200 — a paged KV cache, PagedAttention decode and paged
prefill attention for NVIDIA B200 (sm_100a).

The work is done by ``libpagedkv.so`` (hand-written CUDA kernels plus a C++
host block allocator, C ABI in ``include/paged_kv.h``); this package is its
thin Python binding.  Build the library with
``python -m paged_kv_cache_406_b200.build``.
"""
from .binding import (Allocator, PagedKVError, pkv_append_and_decode, pkv_append_and_decode_fp8,  # noqa: F401
                      pkv_copy_blocks, pkv_decode_workspace_size,
                      pkv_device_status, pkv_kv_append, pkv_kv_append_fp8, pkv_paged_attention_decode,
                      pkv_paged_attention_decode_fp8, pkv_paged_attention_decode_static,
                      pkv_paged_attention_prefill, pkv_prefill_workspace_size, pkv_debug_stall_decode,
                      pkv_debug_stall_prefill,
                      pkv_append_and_decode_pools, pkv_decode_pools_workspace_size,
                      bind_append_and_decode)
from ._native import LIB_PATH, lib  # noqa: F401

__version__ = "1.0.0"
