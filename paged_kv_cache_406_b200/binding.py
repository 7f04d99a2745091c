"""Tensor-level binding: the C entry points under their own names, taking
PyTorch tensors.

Each function checks dtypes, devices, shapes and contiguity, then passes
``data_ptr()`` values and ``torch.cuda.current_stream().cuda_stream`` to the
library.  PyTorch supplies device memory and streams; every step of the
paged-KV path runs in libpagedkv's kernels (device) or allocator (host).
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import _native as N
from ._native import PagedKVError, check, lib

_DTYPES = {torch.float32: N.PKV_F32, torch.bfloat16: N.PKV_BF16, torch.float16: N.PKV_F16,
           torch.float8_e4m3fn: N.PKV_FP8_E4M3, torch.uint8: N.PKV_FP8_E4M3}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}; expected float32, bfloat16, float16 or e4m3 codes")
    return _DTYPES[t.dtype]


def _cuda(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _pool_dims(k_pool: torch.Tensor, v_pool: torch.Tensor):
    if k_pool.dim() != 4 or k_pool.shape != v_pool.shape or k_pool.dtype != v_pool.dtype:
        raise ValueError("k_pool and v_pool must both be [num_blocks, num_kv_heads, block_size, head_dim], same dtype")
    nb, hkv, bs, d = k_pool.shape
    return nb, hkv, bs, d


# ----------------------------------------------------------------------------
# device operations
# ----------------------------------------------------------------------------

def pkv_kv_append(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor,
                  k_pool: torch.Tensor, v_pool: torch.Tensor) -> None:
    """Write each new token's K/V rows into its slot (``slot < 0`` = padding)."""
    nb, hkv, bs, d = _pool_dims(_cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"))
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        _cuda(t, name, k_pool.dtype)
        if t.dim() != 3 or t.shape[1:] != (hkv, d):
            raise ValueError(f"{name} must be [n_tokens, {hkv}, {d}]")
    if k_new.shape != v_new.shape:
        raise ValueError("k_new and v_new differ in shape")
    _cuda(slot_mapping, "slot_mapping", torch.int32)
    if slot_mapping.numel() != k_new.shape[0]:
        raise ValueError("slot_mapping must hold one slot per new token")
    check(lib().pkv_kv_append(k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr(), k_new.shape[0],
                              k_pool.data_ptr(), v_pool.data_ptr(), nb, hkv, d, bs, _dtype_code(k_pool),
                              _stream()))


def pkv_copy_blocks(k_pool: torch.Tensor, v_pool: torch.Tensor, block_pairs: torch.Tensor) -> None:
    """Copy whole blocks src → dst for each ``(src, dst)`` row of ``block_pairs``."""
    nb, hkv, bs, d = _pool_dims(_cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"))
    _cuda(block_pairs, "block_pairs", torch.int32)
    if block_pairs.numel() % 2:
        raise ValueError("block_pairs must be [n_pairs, 2]")
    n = block_pairs.numel() // 2
    check(lib().pkv_copy_blocks(k_pool.data_ptr(), v_pool.data_ptr(), block_pairs.data_ptr(), n, nb, hkv, d, bs,
                                _dtype_code(k_pool), _stream()))


def pkv_decode_workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                              max_blocks_per_seq: int, block_size: int, partition_tokens: int = 0) -> int:
    out = ctypes.c_size_t(0)
    check(lib().pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                                          block_size, partition_tokens, ctypes.byref(out)))
    return out.value


def _new_rows(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor, hkv: int, d: int,
              dtype=None) -> int:
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        _cuda(t, name, dtype)
        if t.dim() != 3 or t.shape[1:] != (hkv, d):
            raise ValueError(f"{name} must be [n_tokens, {hkv}, {d}]")
    if k_new.shape != v_new.shape or k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new differ in shape or dtype")
    _cuda(slot_mapping, "slot_mapping", torch.int32)
    if slot_mapping.numel() != k_new.shape[0]:
        raise ValueError("slot_mapping must hold one slot per new token")
    return k_new.shape[0]


def _decode_io(q: torch.Tensor, hkv: int, d: int, bs: int, block_tables: torch.Tensor, seq_lens: torch.Tensor,
               out: Optional[torch.Tensor], workspace: Optional[torch.Tensor], partition_tokens: int):
    if q.dim() != 3 or q.shape[2] != d:
        raise ValueError(f"q must be [num_seqs, num_q_heads, {d}]")
    B, hq, _ = q.shape
    _cuda(block_tables, "block_tables", torch.int32)
    _cuda(seq_lens, "seq_lens", torch.int32)
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_tables must be [num_seqs, max_blocks_per_seq] and seq_lens [num_seqs]")
    maxb = block_tables.shape[1]
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.float32, device=q.device)
    else:
        _cuda(out, "out", torch.float32)
        if tuple(out.shape) != (B, hq, d):
            raise ValueError("out has the wrong shape")
    need = pkv_decode_workspace_size(B, hq, hkv, d, maxb, bs, partition_tokens)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    else:
        _cuda(workspace, "workspace", torch.uint8)
    return B, hq, maxb, out, workspace


def pkv_paged_attention_decode(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                               block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                               out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                               partition_tokens: int = 0) -> torch.Tensor:
    """PagedAttention decode; returns ``out`` (float32 ``[num_seqs, num_q_heads, head_dim]``)."""
    nb, hkv, bs, d = _pool_dims(_cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"))
    _cuda(q, "q", k_pool.dtype)
    B, hq, maxb, out, workspace = _decode_io(q, hkv, d, bs, block_tables, seq_lens, out, workspace, partition_tokens)
    check(lib().pkv_paged_attention_decode(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                           block_tables.data_ptr(), seq_lens.data_ptr(), B, hq, hkv, d, nb, maxb,
                                           bs, float(scale), _dtype_code(k_pool), partition_tokens,
                                           workspace.data_ptr(), workspace.numel(), out.data_ptr(), _stream()))
    return out


def pkv_append_and_decode(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor, q: torch.Tensor,
                          k_pool: torch.Tensor, v_pool: torch.Tensor, block_tables: torch.Tensor,
                          seq_lens: torch.Tensor, scale: float, out: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, partition_tokens: int = 0) -> torch.Tensor:
    """:func:`pkv_kv_append` then :func:`pkv_paged_attention_decode` in one
    library call (the new rows are written by the launch that plans the
    decode); returns ``out``."""
    nb, hkv, bs, d = _pool_dims(_cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"))
    n = _new_rows(k_new, v_new, slot_mapping, hkv, d, k_pool.dtype)
    _cuda(q, "q", k_pool.dtype)
    B, hq, maxb, out, workspace = _decode_io(q, hkv, d, bs, block_tables, seq_lens, out, workspace, partition_tokens)
    check(lib().pkv_append_and_decode(k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr(), n, q.data_ptr(),
                                      k_pool.data_ptr(), v_pool.data_ptr(), block_tables.data_ptr(),
                                      seq_lens.data_ptr(), B, hq, hkv, d, nb, maxb, bs, float(scale),
                                      _dtype_code(k_pool), partition_tokens, workspace.data_ptr(), workspace.numel(),
                                      out.data_ptr(), _stream()))
    return out


def bind_append_and_decode(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor, q: torch.Tensor,
                           k_pool: torch.Tensor, v_pool: torch.Tensor, block_tables: torch.Tensor,
                           seq_lens: torch.Tensor, scale: float, out: torch.Tensor, workspace: torch.Tensor,
                           partition_tokens: int = 0):
    """:func:`pkv_append_and_decode` checked and marshalled once for a fixed
    set of buffers; returns a callable that issues the call again (on the
    stream current at bind time) with no per-call Python work but the C call
    and its status check.  The buffers must stay alive and keep their shapes;
    their contents may change between calls (a serving loop that stages each
    step's rows and metadata into the same tensors)."""
    nb, hkv, bs, d = _pool_dims(_cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"))
    n = _new_rows(k_new, v_new, slot_mapping, hkv, d, k_pool.dtype)
    _cuda(q, "q", k_pool.dtype)
    B, hq, maxb, out, workspace = _decode_io(q, hkv, d, bs, block_tables, seq_lens, out, workspace, partition_tokens)
    fn = lib().pkv_append_and_decode
    args = (k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr(), n, q.data_ptr(), k_pool.data_ptr(),
            v_pool.data_ptr(), block_tables.data_ptr(), seq_lens.data_ptr(), B, hq, hkv, d, nb, maxb, bs, float(scale),
            _dtype_code(k_pool), partition_tokens, workspace.data_ptr(), workspace.numel(), out.data_ptr(), _stream())
    keep = (k_new, v_new, slot_mapping, q, k_pool, v_pool, block_tables, seq_lens, out, workspace)

    def call():
        rc = fn(*args)
        if rc:
            check(rc)
        return keep[8]

    return call


def pkv_prefill_workspace_size(num_seqs: int, num_kv_heads: int, head_dim: int, max_blocks_per_seq: int,
                               block_size: int, dtype: torch.dtype) -> int:
    """Bytes of the prefill workspace (the f16 copy of V for bf16 pools; 0
    for f16 pools)."""
    out = ctypes.c_size_t(0)
    code = N.PKV_BF16 if dtype == torch.bfloat16 else N.PKV_F16
    check(lib().pkv_prefill_workspace_size(num_seqs, num_kv_heads, head_dim, max_blocks_per_seq, block_size, code,
                                           ctypes.byref(out)))
    return out.value


def pkv_paged_attention_prefill(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                                block_tables: torch.Tensor, seq_lens: torch.Tensor, q_start: torch.Tensor,
                                max_q_len: int, scale: float, out: Optional[torch.Tensor] = None,
                                workspace: Optional[torch.Tensor] = None, stage_v: bool = True) -> torch.Tensor:
    """Causal paged prefill attention; returns ``out`` (float32
    ``[num_q_tokens, num_q_heads, head_dim]``).  Sequence ``b`` owns q rows
    ``q_start[b] .. q_start[b+1]-1`` (int32 ``[num_seqs + 1]`` on the device);
    ``max_q_len`` bounds every chunk length.  For bf16 pools with
    ``stage_v`` the call first copies V into ``workspace`` as f16 (a uint8
    device tensor of :func:`pkv_prefill_workspace_size` bytes, allocated here
    if None) so that P·V runs as one f16 pass; ``stage_v=False`` keeps the
    two bf16 passes (P hi and lo) over the pool's own V."""
    nb, hkv, bs, d = _pool_dims(_cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"))
    _cuda(q, "q", k_pool.dtype)
    if q.dim() != 3 or q.shape[2] != d:
        raise ValueError(f"q must be [num_q_tokens, num_q_heads, {d}]")
    T, hq, _ = q.shape
    _cuda(block_tables, "block_tables", torch.int32)
    _cuda(seq_lens, "seq_lens", torch.int32)
    _cuda(q_start, "q_start", torch.int32)
    B = seq_lens.numel()
    if block_tables.dim() != 2 or block_tables.shape[0] != B or q_start.numel() != B + 1:
        raise ValueError("block_tables must be [num_seqs, max_blocks_per_seq] and q_start [num_seqs + 1]")
    maxb = block_tables.shape[1]
    if out is None:
        out = torch.empty((T, hq, d), dtype=torch.float32, device=q.device)
    else:
        _cuda(out, "out", torch.float32)
        if tuple(out.shape) != (T, hq, d):
            raise ValueError("out has the wrong shape")
    ws_ptr, ws_bytes = None, 0
    if stage_v and k_pool.dtype == torch.bfloat16:
        need = pkv_prefill_workspace_size(B, hkv, d, maxb, bs, k_pool.dtype)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _cuda(workspace, "workspace", torch.uint8)
        if workspace.numel() < need:
            raise ValueError(f"workspace has {workspace.numel()} bytes, {need} needed")
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
    check(lib().pkv_paged_attention_prefill(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                            block_tables.data_ptr(), seq_lens.data_ptr(), q_start.data_ptr(), B, T,
                                            int(max_q_len), hq, hkv, d, nb, maxb, bs, float(scale),
                                            _dtype_code(k_pool), ws_ptr, ws_bytes, out.data_ptr(), _stream()))
    return out


def pkv_paged_attention_decode_static(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                                      block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                                      out: Optional[torch.Tensor] = None, partition_tokens: int = 0) -> torch.Tensor:
    """Decode with the library's static scratch instead of a workspace tensor,
    for callers that cannot allocate device memory while decoding (pass
    ``out`` to allocate nothing here either).  Same result as
    :func:`pkv_paged_attention_decode`; calls overlapping on the GPU race on
    the shared scratch."""
    nb, hkv, bs, d = _pool_dims(_cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"))
    _cuda(q, "q", k_pool.dtype)
    if q.dim() != 3 or q.shape[2] != d:
        raise ValueError(f"q must be [num_seqs, num_q_heads, {d}]")
    B, hq, _ = q.shape
    _cuda(block_tables, "block_tables", torch.int32)
    _cuda(seq_lens, "seq_lens", torch.int32)
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_tables must be [num_seqs, max_blocks_per_seq] and seq_lens [num_seqs]")
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.float32, device=q.device)
    else:
        _cuda(out, "out", torch.float32)
        if tuple(out.shape) != (B, hq, d):
            raise ValueError("out has the wrong shape")
    check(lib().pkv_paged_attention_decode_static(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                                  block_tables.data_ptr(), seq_lens.data_ptr(), B, hq, hkv, d, nb,
                                                  block_tables.shape[1], bs, float(scale), _dtype_code(k_pool),
                                                  partition_tokens, out.data_ptr(), _stream()))
    return out


def _fp8_pool(t: torch.Tensor, name: str) -> torch.Tensor:
    _cuda(t, name)
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError(f"{name} must hold e4m3 codes (torch.uint8 or torch.float8_e4m3fn), got {t.dtype}")
    return t


def pkv_kv_append_fp8(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor, k_pool: torch.Tensor,
                      v_pool: torch.Tensor, k_scale: float, v_scale: float) -> None:
    """Quantise each new token's K/V rows to e4m3 (x / scale, nearest, saturating)
    and write them into their slots of the e4m3 pools."""
    _fp8_pool(k_pool, "k_pool")
    _fp8_pool(v_pool, "v_pool")
    if k_pool.dim() != 4 or k_pool.shape != v_pool.shape:
        raise ValueError("pools must be [num_blocks, num_kv_heads, block_size, head_dim]")
    nb, hkv, bs, d = k_pool.shape
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        _cuda(t, name)
        if t.dim() != 3 or t.shape[1:] != (hkv, d):
            raise ValueError(f"{name} must be [n_tokens, {hkv}, {d}]")
    if k_new.shape != v_new.shape or k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new differ in shape or dtype")
    _cuda(slot_mapping, "slot_mapping", torch.int32)
    if slot_mapping.numel() != k_new.shape[0]:
        raise ValueError("slot_mapping must hold one slot per new token")
    check(lib().pkv_kv_append_fp8(k_new.data_ptr(), v_new.data_ptr(), _dtype_code(k_new), slot_mapping.data_ptr(),
                                  k_new.shape[0], k_pool.data_ptr(), v_pool.data_ptr(), nb, hkv, d, bs,
                                  float(k_scale), float(v_scale), _stream()))


def pkv_paged_attention_decode_fp8(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                                   block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float, k_scale: float,
                                   v_scale: float, out: Optional[torch.Tensor] = None,
                                   workspace: Optional[torch.Tensor] = None, partition_tokens: int = 0) -> torch.Tensor:
    """PagedAttention decode over e4m3 pools (q float16); float32 output."""
    _fp8_pool(k_pool, "k_pool")
    _fp8_pool(v_pool, "v_pool")
    if k_pool.dim() != 4 or k_pool.shape != v_pool.shape:
        raise ValueError("pools must be [num_blocks, num_kv_heads, block_size, head_dim]")
    nb, hkv, bs, d = k_pool.shape
    _cuda(q, "q", torch.float16)
    B, hq, maxb, out, workspace = _decode_io(q, hkv, d, bs, block_tables, seq_lens, out, workspace, partition_tokens)
    check(lib().pkv_paged_attention_decode_fp8(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                               block_tables.data_ptr(), seq_lens.data_ptr(), B, hq, hkv, d, nb, maxb,
                                               bs, float(scale), float(k_scale), float(v_scale), partition_tokens,
                                               workspace.data_ptr(), workspace.numel(), out.data_ptr(), _stream()))
    return out


def pkv_append_and_decode_fp8(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor,
                              q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                              block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float, k_scale: float,
                              v_scale: float, out: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None, partition_tokens: int = 0) -> torch.Tensor:
    """:func:`pkv_kv_append_fp8` then :func:`pkv_paged_attention_decode_fp8`
    in one library call; returns ``out``."""
    _fp8_pool(k_pool, "k_pool")
    _fp8_pool(v_pool, "v_pool")
    if k_pool.dim() != 4 or k_pool.shape != v_pool.shape:
        raise ValueError("pools must be [num_blocks, num_kv_heads, block_size, head_dim]")
    nb, hkv, bs, d = k_pool.shape
    n = _new_rows(k_new, v_new, slot_mapping, hkv, d)
    _cuda(q, "q", torch.float16)
    B, hq, maxb, out, workspace = _decode_io(q, hkv, d, bs, block_tables, seq_lens, out, workspace, partition_tokens)
    check(lib().pkv_append_and_decode_fp8(k_new.data_ptr(), v_new.data_ptr(), _dtype_code(k_new),
                                          slot_mapping.data_ptr(), n, q.data_ptr(), k_pool.data_ptr(),
                                          v_pool.data_ptr(), block_tables.data_ptr(), seq_lens.data_ptr(), B, hq, hkv,
                                          d, nb, maxb, bs, float(scale), float(k_scale), float(v_scale),
                                          partition_tokens, workspace.data_ptr(), workspace.numel(), out.data_ptr(),
                                          _stream()))
    return out


def _pool_array(pools):
    """ctypes array of pkv_pool_t from (k_pool, v_pool, block_tables, num_seqs) tuples."""
    arr = (N.pkv_pool_t * len(pools))()
    for c, (k_pool, v_pool, tables, n) in enumerate(pools):
        nb, _, bs, _ = _pool_dims(_cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"))
        _cuda(tables, "block_tables", torch.int32)
        if tables.dim() != 2 or tables.shape[0] < n:
            raise ValueError("each pool's block_tables must be [num_seqs, max_blocks_per_seq]")
        arr[c] = N.pkv_pool_t(k_pool.data_ptr(), v_pool.data_ptr(), tables.data_ptr(), nb, bs, tables.shape[1], int(n))
    return arr


def pkv_decode_pools_workspace_size(pools, num_q_heads: int, partition_tokens: int = 0) -> int:
    """Workspace bytes of :func:`pkv_append_and_decode_pools` for ``pools``."""
    arr = _pool_array(pools)
    _, hkv, _, d = pools[0][0].shape
    out = ctypes.c_size_t(0)
    check(lib().pkv_decode_pools_workspace_size(arr, len(pools), num_q_heads, hkv, d, partition_tokens,
                                                ctypes.byref(out)))
    return out.value


def pkv_append_and_decode_pools(pools, k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor,
                                q: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                                out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                                partition_tokens: int = 0) -> torch.Tensor:
    """One decode step (append + attention) over a batch spread across
    pools of different block sizes.  ``pools``: up to 3 tuples
    ``(k_pool, v_pool, block_tables, num_seqs)``; the rows of ``k_new``,
    ``v_new``, ``slot_mapping`` (pool-local slots), ``q`` and ``seq_lens``
    follow the pools' sequences in pool order."""
    arr = _pool_array(pools)
    n = sum(int(x[3]) for x in pools)
    _, hkv, _, d = pools[0][0].shape
    _cuda(q, "q", pools[0][0].dtype)
    if q.dim() != 3 or q.shape[0] != n or q.shape[2] != d:
        raise ValueError(f"q must be [{n}, num_q_heads, {d}]")
    hq = q.shape[1]
    for t, name in ((k_new, "k_new"), (v_new, "v_new")):
        _cuda(t, name, pools[0][0].dtype)
        if tuple(t.shape) != (n, hkv, d):
            raise ValueError(f"{name} must be [{n}, {hkv}, {d}]")
    _cuda(slot_mapping, "slot_mapping", torch.int32)
    _cuda(seq_lens, "seq_lens", torch.int32)
    if slot_mapping.numel() != n or seq_lens.numel() != n:
        raise ValueError(f"slot_mapping and seq_lens must have {n} entries")
    need = pkv_decode_pools_workspace_size(pools, hq, partition_tokens)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _cuda(workspace, "workspace", torch.uint8)
    if out is None:
        out = torch.empty((n, hq, d), dtype=torch.float32, device=q.device)
    _cuda(out, "out", torch.float32)
    if tuple(out.shape) != (n, hq, d):
        raise ValueError("out has the wrong shape")
    check(lib().pkv_append_and_decode_pools(arr, len(pools), k_new.data_ptr(), v_new.data_ptr(),
                                            slot_mapping.data_ptr(), q.data_ptr(), seq_lens.data_ptr(), hq, hkv, d,
                                            float(scale), _dtype_code(pools[0][0]), partition_tokens,
                                            workspace.data_ptr(), workspace.numel(), out.data_ptr(), _stream()))
    return out


def pkv_device_status(clear: bool = True) -> int:
    """Synchronise the current stream and return the device status word."""
    st = ctypes.c_int32(0)
    check(lib().pkv_device_status(_stream(), ctypes.byref(st), 1 if clear else 0))
    return st.value


def pkv_debug_stall_decode(cta: int = -1) -> None:
    """Test support for the bounded waits: the decode launches that follow
    leave CTA ``cta``'s first work unit without copies, so its consumers'
    waits run out (after the normal limit); ``cta < 0`` restores normal
    operation."""
    check(lib().pkv_debug_stall_decode(int(cta)))


def pkv_debug_stall_prefill(cta: int = -1) -> None:
    """Test support for the prefill kernel's bounded waits: in the prefill
    launches that follow, the K producer of CTA ``cta`` skips its first
    chunk, so the MMA warp's wait for it runs out (after the normal limit);
    ``cta < 0`` restores normal operation."""
    check(lib().pkv_debug_stall_prefill(int(cta)))


# ----------------------------------------------------------------------------
# host block allocator
# ----------------------------------------------------------------------------

def _i64_array(ids: Sequence[int]):
    a = np.ascontiguousarray(np.asarray(ids, dtype=np.int64))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


class Allocator:
    """The library's host block allocator (pkv_alloc_*): free stack, refcounts,
    copy-on-write; every failing call leaves it unchanged."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self._h = ctypes.c_void_p()
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        if free_order is not None:
            fo = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            if fo.size != num_blocks:
                raise ValueError("free_order must list every block once")
            ptr = fo.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        else:
            ptr = None
        check(lib().pkv_alloc_create(num_blocks, block_size, ptr, ctypes.byref(self._h)))
        self._slot_buf = np.zeros(0, dtype=np.int32)
        self._cow_buf = np.zeros(0, dtype=np.int32)

    def close(self) -> None:
        if self._h:
            lib().pkv_alloc_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add(self, seq_id: int, n_tokens: int) -> None:
        check(lib().pkv_seq_add(self._h, seq_id, n_tokens))

    def add_cached(self, seq_id: int, tokens) -> int:
        """Admit a sequence with known prompt token ids, reusing cached blocks of
        an identical prefix; returns the number of leading tokens already cached."""
        t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = ctypes.c_int32(0)
        check(lib().pkv_seq_add_cached(self._h, seq_id, t.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), t.size,
                                       ctypes.byref(n)))
        return n.value

    def fork(self, parent: int, child: int) -> None:
        check(lib().pkv_seq_fork(self._h, parent, child))

    def free(self, seq_id: int) -> None:
        check(lib().pkv_seq_free(self._h, seq_id))

    def seq_len(self, seq_id: int) -> int:
        n = ctypes.c_int32(0)
        check(lib().pkv_seq_len(self._h, seq_id, ctypes.byref(n)))
        return n.value

    def append_slots(self, seq_ids: Sequence[int], slot_out: Optional[np.ndarray] = None):
        """Reserve one slot per sequence; returns ``(slots int32[n], cow_pairs int32[k, 2])``."""
        ids, ip = _i64_array(seq_ids)
        n = ids.size
        if slot_out is None:
            slot_out = np.empty(n, dtype=np.int32)
        if self._cow_buf.size < 2 * n:
            self._cow_buf = np.empty(2 * max(n, 1), dtype=np.int32)
        ncow = ctypes.c_int32(0)
        check(lib().pkv_seq_append_slots(self._h, ip, n, slot_out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                         self._cow_buf.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n,
                                         ctypes.byref(ncow)))
        return slot_out, self._cow_buf[: 2 * ncow.value].reshape(-1, 2).copy()

    def block_tables(self, seq_ids: Sequence[int], max_blocks: int, tables_out=None, seq_lens_out=None):
        """``(tables int32[n, max_blocks] padded with -1, seq_lens int32[n])``."""
        ids, ip = _i64_array(seq_ids)
        n = ids.size
        if tables_out is None:
            tables_out = np.empty((n, max_blocks), dtype=np.int32)
        if seq_lens_out is None:
            seq_lens_out = np.empty(n, dtype=np.int32)
        check(lib().pkv_block_tables(self._h, ip, n, max_blocks,
                                     tables_out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                     seq_lens_out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))))
        return tables_out, seq_lens_out

    def stats(self) -> dict:
        s = N.pkv_stats_t()
        check(lib().pkv_alloc_stats(self._h, ctypes.byref(s)))
        return {name: getattr(s, name) for name, _ in s._fields_}


__all__ = ["Allocator", "PagedKVError", "pkv_kv_append", "pkv_copy_blocks", "pkv_decode_workspace_size",
           "pkv_paged_attention_decode", "pkv_paged_attention_decode_static", "pkv_device_status",
           "pkv_debug_stall_decode", "pkv_debug_stall_prefill", "pkv_paged_attention_prefill", "pkv_prefill_workspace_size",
           "pkv_append_and_decode_pools", "pkv_decode_pools_workspace_size", "bind_append_and_decode",
           "pkv_kv_append_fp8", "pkv_paged_attention_decode_fp8", "pkv_append_and_decode",
           "pkv_append_and_decode_fp8"]
