"""ctypes binding of libpagedkv.so (argument marshalling only).

Every function here has the name of the C entry point it calls and forwards
raw pointers, sizes and the current CUDA stream; all computation happens in
the library's kernels and host allocator.  Loading fails loudly when the
library has not been built: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpagedkv.so")

PKV_OK = 0
PKV_ERR_INVALID_ARG = -1
PKV_ERR_OUT_OF_BLOCKS = -2
PKV_ERR_UNKNOWN_SEQ = -3
PKV_ERR_UNSUPPORTED = -4
PKV_ERR_CUDA = -5
PKV_ERR_DEVICE_TIMEOUT = -6
PKV_ERR_SEQ_EXISTS = -7
PKV_ERR_BAD_BLOCK = -8

PKV_F32, PKV_BF16, PKV_F16, PKV_FP8_E4M3 = 0, 1, 2, 3

# Every entry point include/paged_kv.h declares, with its ctypes signature.
_i32, _i64, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_pi32 = ctypes.POINTER(ctypes.c_int32)
_pi64 = ctypes.POINTER(ctypes.c_int64)


class pkv_stats_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "num_blocks", "block_size", "free_blocks", "used_blocks", "num_seqs", "cow_copies",
        "logical_tokens", "waste_tokens", "cached_blocks", "cache_queries", "cache_hits")]


class pkv_pool_t(ctypes.Structure):
    """One pool of a batch spread over several pools (pkv_append_and_decode_pools)."""
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("block_tables", ctypes.c_void_p),
                ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_seqs", ctypes.c_int32)]


_ppool = ctypes.POINTER(pkv_pool_t)

SIGNATURES = {
    "pkv_last_error_string": (ctypes.c_char_p, []),
    "pkv_version": (ctypes.c_char_p, []),
    "pkv_alloc_create": (ctypes.c_int, [_i32, _i32, _pi32, ctypes.POINTER(_vp)]),
    "pkv_alloc_destroy": (None, [_vp]),
    "pkv_seq_add": (ctypes.c_int, [_vp, _i64, _i32]),
    "pkv_seq_fork": (ctypes.c_int, [_vp, _i64, _i64]),
    "pkv_seq_add_cached": (ctypes.c_int, [_vp, _i64, _pi32, _i32, _pi32]),
    "pkv_seq_append_slots": (ctypes.c_int, [_vp, _pi64, _i32, _pi32, _pi32, _i32, _pi32]),
    "pkv_seq_free": (ctypes.c_int, [_vp, _i64]),
    "pkv_seq_len": (ctypes.c_int, [_vp, _i64, _pi32]),
    "pkv_block_tables": (ctypes.c_int, [_vp, _pi64, _i32, _i32, _pi32, _pi32]),
    "pkv_alloc_stats": (ctypes.c_int, [_vp, ctypes.POINTER(pkv_stats_t)]),
    "pkv_kv_append": (ctypes.c_int, [_vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pkv_copy_blocks": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pkv_decode_workspace_size": (ctypes.c_int, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]),
    "pkv_paged_attention_decode": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                                  _i32, _f32, _i32, _i32, _vp, _sz, _vp, _vp]),
    "pkv_device_status": (ctypes.c_int, [_vp, _pi32, _i32]),
    "pkv_debug_stall_decode": (ctypes.c_int, [_i32]),
    "pkv_debug_stall_prefill": (ctypes.c_int, [_i32]),
    "pkv_paged_attention_decode_static": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                                         _i32, _i32, _f32, _i32, _i32, _vp, _vp]),
    "pkv_static_workspace_bytes": (ctypes.c_size_t, []),
    "pkv_kv_append_fp8": (ctypes.c_int, [_vp, _vp, _i32, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _f32, _f32,
                                         _vp]),
    "pkv_paged_attention_decode_fp8": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                                      _i32, _f32, _f32, _f32, _i32, _vp, _sz, _vp, _vp]),
    "pkv_append_and_decode": (ctypes.c_int, [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                             _i32, _i32, _i32, _f32, _i32, _i32, _vp, _sz, _vp, _vp]),
    "pkv_append_and_decode_fp8": (ctypes.c_int, [_vp, _vp, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                                 _i32, _i32, _i32, _i32, _f32, _f32, _f32, _i32, _vp, _sz, _vp, _vp]),
    "pkv_step_meta_bytes": (ctypes.c_size_t, [_i32, _i32]),
    # seq_ids (const int64_t*) as a plain address: the per-step caller passes
    # the int64 array's address without building a ctypes pointer object
    "pkv_decode_step_host": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32,
                                            _i32, _f32, _f32, _i32, _vp, _sz, _vp]),
    "pkv_paged_attention_prefill": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                                   _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp]),
    "pkv_prefill_workspace_size": (ctypes.c_int, [_i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]),
    "pkv_decode_pools_workspace_size": (ctypes.c_int, [_ppool, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]),
    "pkv_append_and_decode_pools": (ctypes.c_int, [_ppool, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _f32, _i32,
                                                   _i32, _vp, _sz, _vp, _vp]),
}


class StepBuffers(ctypes.Structure):
    """pkv_step_buffers_t: the host and device buffers of one pkv_decode_step_host call."""
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "meta_host", "meta_dev", "q_host", "k_host", "v_host", "q_dev", "k_dev", "v_dev", "out_dev", "out_host",
        "wait_event", "done_event", "h2d_stream", "d2h_stream", "compute_done", "d2h_done")]


class PagedKVError(RuntimeError):
    """A libpagedkv call returned a negative status."""

    def __init__(self, code: int, message: str):
        super().__init__(f"[{code}] {message}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_406_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(rc: int) -> None:
    if rc != PKV_OK:
        raise PagedKVError(rc, lib().pkv_last_error_string().decode(errors="replace"))
