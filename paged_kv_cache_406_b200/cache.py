"""PagedKVCache: one layer's paged K/V pools on a GPU plus the host allocator,
and the decode step that ties them together.

One call of :meth:`PagedKVCache.decode_step` is the whole hot path of a decode
step for one layer ("vLLM's 'memory paging' — PagedAttention illustrated", §3):

1. slot reservation on the host (pkv_seq_append_slots): a new block when the
   last one is full, a private copy when it is shared;
2. one host→device copy of the step's metadata (slots, copy pairs, block
   tables, lengths) from pinned memory;
3. pkv_copy_blocks for the copy-on-write pairs, if any;
4. pkv_append_and_decode: the new tokens' K/V written into their slots by the
   launch that plans the decode, then PagedAttention decode (plus its
   partition merge) over every sequence, new token included.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import binding as B
from ._native import StepBuffers, check, lib


class PagedKVCache:
    def __init__(self, num_blocks: int, num_kv_heads: int, head_dim: int, block_size: int,
                 dtype: torch.dtype, max_blocks_per_seq: int, device="cuda", free_order=None,
                 k_pool: Optional[torch.Tensor] = None, v_pool: Optional[torch.Tensor] = None,
                 k_scale: float = 1.0, v_scale: float = 1.0):
        """``dtype`` torch.float8_e4m3fn (or torch.uint8) keeps the pools as e4m3
        codes with per-pool scales ``k_scale`` / ``v_scale`` (the overview page's
        FP8 KV cache); new rows are quantised on append and q must be float16."""
        self.device = torch.device(device)
        self.fp8 = dtype in (torch.float8_e4m3fn, torch.uint8)
        self.k_scale, self.v_scale = float(k_scale), float(v_scale)
        self.num_blocks, self.num_kv_heads = int(num_blocks), int(num_kv_heads)
        self.head_dim, self.block_size = int(head_dim), int(block_size)
        self.dtype = dtype
        self.max_blocks = int(max_blocks_per_seq)
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k_pool = k_pool if k_pool is not None else torch.empty(shape, dtype=dtype, device=self.device)
        self.v_pool = v_pool if v_pool is not None else torch.empty(shape, dtype=dtype, device=self.device)
        if tuple(self.k_pool.shape) != shape or tuple(self.v_pool.shape) != shape:
            raise ValueError(f"pools must be {shape}")
        self.alloc = B.Allocator(num_blocks, block_size, free_order)
        self._meta_cap = 0
        self._ws = None
        self._out = None

    # -- sequence lifecycle (host) -----------------------------------------
    def add(self, seq_id: int, n_tokens: int) -> None:
        self.alloc.add(seq_id, n_tokens)

    def add_cached(self, seq_id: int, tokens) -> int:
        """Admit a sequence by its token ids, reusing cached full blocks of its
        prefix; returns how many leading tokens already sit in the pool (the
        caller writes K/V only for the rest)."""
        return self.alloc.add_cached(seq_id, tokens)

    def fork(self, parent: int, child: int) -> None:
        self.alloc.fork(parent, child)

    def free(self, seq_id: int) -> None:
        self.alloc.free(seq_id)

    # -- metadata staging ----------------------------------------------------
    def _ensure_meta(self, n: int) -> None:
        # layout (int32): slots[n] | seq_lens[n] | cow[2n] | tables[n * max_blocks]
        need = n * (4 + self.max_blocks)
        if need <= self._meta_cap:
            return
        self._meta_host = torch.empty(need, dtype=torch.int32, pin_memory=True)
        self._meta_dev = torch.empty(need, dtype=torch.int32, device=self.device)
        self._meta_np = self._meta_host.numpy()
        self._meta_cap = need
        self._h2d_done = None

    def prepare_step(self, seq_ids: Sequence[int]):
        """Host part of a decode step: reserve slots and build the metadata
        (numpy views into pinned memory).  Returns ``(n_cow, views)``."""
        n = len(seq_ids)
        self._ensure_meta(n)
        if self._h2d_done is not None:
            self._h2d_done.synchronize()  # the previous copy no longer reads the pinned buffer
        m = self._meta_np
        slots = m[:n]
        lens = m[n:2 * n]
        cow = m[2 * n:4 * n]
        tables = m[4 * n:4 * n + n * self.max_blocks].reshape(n, self.max_blocks)
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        ip = ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
        ncow = ctypes.c_int32(0)
        i32p = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))  # noqa: E731
        check(lib().pkv_seq_append_slots(self.alloc._h, ip, n, i32p(slots), i32p(cow), n, ctypes.byref(ncow)))
        check(lib().pkv_block_tables(self.alloc._h, ip, n, self.max_blocks, i32p(tables), i32p(lens)))
        return ncow.value, (slots, lens, cow, tables)

    def upload_step(self, n: int):
        """Copy the staged metadata to the device; returns device views."""
        used = n * (4 + self.max_blocks)
        self._meta_dev[:used].copy_(self._meta_host[:used], non_blocking=True)
        ev = torch.cuda.Event()
        ev.record()
        self._h2d_done = ev
        d = self._meta_dev
        return (d[:n], d[n:2 * n], d[2 * n:4 * n], d[4 * n:4 * n + n * self.max_blocks].view(n, self.max_blocks))

    def _buffers(self, n: int, num_q_heads: int, partition_tokens: int):
        ws = B.pkv_decode_workspace_size(n, num_q_heads, self.num_kv_heads, self.head_dim, self.max_blocks,
                                         self.block_size, partition_tokens)
        if self._ws is None or self._ws.numel() < ws:
            self._ws = torch.empty(ws, dtype=torch.uint8, device=self.device)
        shape = (n, num_q_heads, self.head_dim)
        if self._out is None or tuple(self._out.shape) != shape:
            self._out = torch.empty(shape, dtype=torch.float32, device=self.device)
        return self._ws, self._out

    # -- the decode step -----------------------------------------------------
    def decode_step(self, seq_ids: Sequence[int], q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                    scale: float, partition_tokens: int = 0, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Append one token per sequence and attend over every cached token.

        ``q`` [n, Hq, D], ``k_new``/``v_new`` [n, Hkv, D] in the pool dtype, on
        the device or in (pinned) host memory.  Returns float32 [n, Hq, D] on
        the device: ``out`` if given (a contiguous device tensor), else a
        buffer of this cache valid until the next step."""
        n = len(seq_ids)
        ncow, _ = self.prepare_step(seq_ids)
        slots, lens, cow, tables = self.upload_step(n)
        q, k_new, v_new = (t.to(self.device, non_blocking=True) for t in (q, k_new, v_new))
        if ncow:
            B.pkv_copy_blocks(self.k_pool, self.v_pool, cow[:2 * ncow].view(ncow, 2))
        ws, own = self._buffers(n, q.shape[1], partition_tokens)
        out = own if out is None else out
        if self.fp8:
            return B.pkv_append_and_decode_fp8(k_new, v_new, slots, q, self.k_pool, self.v_pool, tables, lens, scale,
                                               self.k_scale, self.v_scale, out=out, workspace=ws,
                                               partition_tokens=partition_tokens)
        return B.pkv_append_and_decode(k_new, v_new, slots, q, self.k_pool, self.v_pool, tables, lens, scale,
                                       out=out, workspace=ws, partition_tokens=partition_tokens)

    # -- the decode step in one library call -------------------------------
    def decode_step_host(self, seq_ids: np.ndarray, q_host: torch.Tensor, k_host: torch.Tensor,
                         v_host: torch.Tensor, scale: float, out_host: Optional[torch.Tensor] = None,
                         partition_tokens: int = 0, overlap: bool = True) -> torch.Tensor:
        """The decode step of :meth:`decode_step` as one pkv_decode_step_host
        call: slot reservation, metadata and row copies from host memory,
        copy-on-write, append, attention and (with ``out_host``) the copy of
        the result back to the host.  ``seq_ids``: int64 numpy array;
        ``q_host`` [n, Hq, D], ``k_host`` / ``v_host`` [n, Hkv, D] pinned host
        tensors (float16 for e4m3 pools, else the pool dtype).  Two metadata
        staging buffers alternate, so a step only waits for the copy two steps
        back before overwriting one.  Returns the device output (valid until
        the next step) or ``out_host``.  With ``overlap`` the host-to-device
        and device-to-host copies run on two copy streams of this cache, so
        they proceed under the neighbouring steps' kernels (two sets of device
        buffers alternate); ``out_host`` is then complete once the current
        stream and the copy streams have been synchronised."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = int(ids.size)
        hq = q_host.shape[1]
        self._ensure_step(n, hq)
        k = self._step_k
        self._step_k ^= 1
        # the call's fixed arguments for the step buffers' capacity and this
        # partition size (a workspace sized for the capacity serves every
        # smaller batch), recomputed when either changes
        key = (self._step_key, int(partition_tokens))
        fixed = getattr(self, "_step_fixed", None)
        if fixed is None or fixed[0] != key:
            need = B.pkv_decode_workspace_size(self._step_key[0], hq, self.num_kv_heads, self.head_dim,
                                               self.max_blocks, self.block_size, partition_tokens)
            ws = torch.empty(max(1, need), dtype=torch.uint8, device=self.device)
            head = (self.k_pool.data_ptr(), self.v_pool.data_ptr(), self.num_blocks, hq, self.num_kv_heads,
                    self.head_dim, self.block_size, self.max_blocks)
            tail = (B._dtype_code(self.k_pool), self.k_scale, self.v_scale, int(partition_tokens), ws.data_ptr(),
                    ws.numel())
            dev = self.device.index if self.device.index is not None else torch.cuda.current_device()
            fixed = (key, (head, tail, dev, ws))  # holds ws: its address stays valid while cached
            self._step_fixed = fixed
        fixed = fixed[1]
        head, tail, dev, _ = fixed
        b = self._step_bufs[k]
        out = self._step_out[k][:n]
        b.q_host, b.k_host, b.v_host = q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr()
        b.out_host = out_host.data_ptr() if out_host is not None else None
        b.h2d_stream = self._h2d_stream.cuda_stream if overlap else None
        b.d2h_stream = self._d2h_stream.cuda_stream if overlap else None
        check(lib().pkv_decode_step_host(
            self.alloc._h, ids.ctypes.data, n, ctypes.byref(b), *head, float(scale), *tail,
            torch._C._cuda_getCurrentRawStream(dev)))
        return out_host if out_host is not None else out

    def wait_copies(self) -> None:
        """Makes the current stream wait for the copies that
        :meth:`decode_step_host` issued on this cache's copy streams (with
        ``overlap``), so that work recorded next on the current stream - a
        timing event, a read of ``out_host`` after synchronising it - comes
        after the last result has reached the host."""
        cur = torch.cuda.current_stream(self.device)
        for st in (getattr(self, "_h2d_stream", None), getattr(self, "_d2h_stream", None)):
            if st is not None:
                cur.wait_stream(st)

    def _ensure_step(self, n: int, hq: int) -> None:
        # buffers sized by capacity: a batch of up to the largest n seen so far
        # reuses them; a larger one (or another head count) allocates anew,
        # after the device has finished with the old ones (copies in flight on
        # the copy streams read and write them)
        cap = getattr(self, "_step_key", None)
        if cap is not None and cap[1] == hq and n <= cap[0]:
            return
        if cap is not None:
            torch.cuda.synchronize(self.device)
        n = max(n, cap[0] if cap is not None else 0)
        key = (n, hq)
        nbytes = int(lib().pkv_step_meta_bytes(n, self.max_blocks))
        io = torch.float16 if self.fp8 else self.dtype
        self._step_hold = []
        self._step_bufs = []
        self._step_out = []
        self._h2d_stream = torch.cuda.Stream(self.device)
        self._d2h_stream = torch.cuda.Stream(self.device)
        # per buffer set: copies in done (host may rewrite the staging), kernels
        # done (the set's device buffers may be rewritten), copy back done
        self._step_events = [[torch.cuda.Event() for _ in range(3)] for _ in range(2)]
        for k in range(2):
            mh = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
            md = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            qd = torch.empty((n, hq, self.head_dim), dtype=io, device=self.device)
            kd = torch.empty((n, self.num_kv_heads, self.head_dim), dtype=io, device=self.device)
            vd = torch.empty_like(kd)
            od = torch.empty((n, hq, self.head_dim), dtype=torch.float32, device=self.device)
            self._step_hold += [mh, md, qd, kd, vd]
            self._step_out.append(od)
            for ev in self._step_events[k]:
                ev.record()  # completed events: the first waits return at once
            h2d, kern, d2h = (ev.cuda_event for ev in self._step_events[k])
            b = StepBuffers(meta_host=mh.data_ptr(), meta_dev=md.data_ptr(), q_dev=qd.data_ptr(),
                            k_dev=kd.data_ptr(), v_dev=vd.data_ptr(), out_dev=od.data_ptr(),
                            wait_event=h2d, done_event=h2d, compute_done=kern, d2h_done=d2h)
            self._step_bufs.append(b)
        self._step_k = 0
        self._step_key = key

    def stats(self) -> dict:
        return self.alloc.stats()


def block_size_for(seq_len: int) -> int:
    """The optimisation-overview page's block-size classes (§3.3): 32 below
    1024 tokens, 16 from 1024 to below 8192, 8 from 8192 on."""
    if seq_len < 1024:
        return 32
    if seq_len < 8192:
        return 16
    return 8


class AdaptivePagedKVCache:
    """Adaptive block size (optimisation-overview page §3.3): one paged pool
    per block-size class (32, 16, 8 tokens); a sequence joins the class of
    its length at admission and keeps it for life (the page leaves migration
    open; none is done).  A decode step serves every class in one call
    (pkv_append_and_decode_pools), or one call per class.

    ``seq_ids`` passed to :meth:`decode_step` must be grouped by class in the
    order 32, 16, 8 (:meth:`order` returns live ids that way), so that each
    class works on a contiguous slice of q, the new rows and the output."""

    CLASSES = (32, 16, 8)

    def __init__(self, blocks_per_class: dict, num_kv_heads: int, head_dim: int, dtype: torch.dtype,
                 max_tokens: int, device="cuda", seed: int = 0):
        self.caches = {}
        for bs in self.CLASSES:
            nb = int(blocks_per_class.get(bs, 0))
            if nb <= 0:
                continue
            order = np.random.Generator(np.random.PCG64(seed + bs)).permutation(nb).astype(np.int32)
            self.caches[bs] = PagedKVCache(nb, num_kv_heads, head_dim, bs, dtype, -(-max_tokens // bs),
                                           device=device, free_order=order)
        self.cls: dict = {}

    def add(self, seq_id: int, n_tokens: int) -> int:
        bs = block_size_for(n_tokens)
        if bs not in self.caches:
            raise ValueError(f"no pool for block size {bs}")
        self.caches[bs].add(seq_id, n_tokens)
        self.cls[seq_id] = bs
        return bs

    def free(self, seq_id: int) -> None:
        self.caches[self.cls.pop(seq_id)].free(seq_id)

    def order(self) -> list:
        return [s for bs in self.CLASSES for s in self.cls if self.cls[s] == bs]

    def decode_step(self, seq_ids: Sequence[int], q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                    scale: float, out: Optional[torch.Tensor] = None, one_call: bool = True) -> torch.Tensor:
        """Append one token per sequence and attend, over every class.  With
        ``one_call`` (16-bit pools, head_dim 128, 2 to 8 query heads per KV
        head) the classes share one pkv_append_and_decode_pools call (one
        append + plan, decode and merge launch for the whole batch); otherwise
        each class runs its own decode step."""
        n = len(seq_ids)
        ranks = [self.CLASSES.index(self.cls[s]) for s in seq_ids]
        if any(a > b for a, b in zip(ranks, ranks[1:])):
            raise ValueError("seq_ids must be grouped by block-size class (32, 16, 8)")
        dev = next(iter(self.caches.values())).device
        if out is None:
            out = torch.empty((n, q.shape[1], q.shape[2]), dtype=torch.float32, device=dev)
        counts = [sum(1 for r in ranks if self.CLASSES[r] == bs) for bs in self.CLASSES]
        any_cache = next(iter(self.caches.values()))
        g = q.shape[1] // any_cache.num_kv_heads
        if not (one_call and any_cache.dtype in (torch.bfloat16, torch.float16) and any_cache.head_dim == 128
                and g in (2, 4, 8)):
            a = 0
            for bs, m in zip(self.CLASSES, counts):
                if m:
                    self.caches[bs].decode_step(seq_ids[a:a + m], q[a:a + m], k_new[a:a + m], v_new[a:a + m],
                                                scale, out=out[a:a + m])
                a += m
            return out
        # host: slots, copy-on-write and tables per class; the step's slots and
        # lengths gathered into one pinned buffer and copied up once
        if getattr(self, "_sl_cap", 0) < n:
            self._sl_host = torch.empty(2 * n, dtype=torch.int32, pin_memory=True)
            self._sl_dev = torch.empty(2 * n, dtype=torch.int32, device=dev)
            self._sl_cap = n
            self._sl_done = None
        if self._sl_done is not None:
            self._sl_done.synchronize()
        sl = self._sl_host.numpy()
        pools, a = [], 0
        for bs, m in zip(self.CLASSES, counts):
            if bs not in self.caches:
                continue
            c = self.caches[bs]
            if not m:  # a class with no sequence this step: a pool of none
                pools.append((c.k_pool, c.v_pool, torch.empty((0, c.max_blocks), dtype=torch.int32, device=dev), 0))
                continue
            ncow, (slots, lens, _, _) = c.prepare_step(seq_ids[a:a + m])
            sl[a:a + m] = slots[:m]
            sl[n + a:n + a + m] = lens[:m]
            _, _, cow, tables = c.upload_step(m)
            if ncow:
                B.pkv_copy_blocks(c.k_pool, c.v_pool, cow[:2 * ncow].view(ncow, 2))
            pools.append((c.k_pool, c.v_pool, tables, m))
            a += m
        self._sl_dev[:2 * n].copy_(self._sl_host[:2 * n], non_blocking=True)
        ev = torch.cuda.Event()
        ev.record()
        self._sl_done = ev
        q, k_new, v_new = (t.to(dev, non_blocking=True) for t in (q, k_new, v_new))
        ws = getattr(self, "_pool_ws", None)
        need = B.pkv_decode_pools_workspace_size(pools, q.shape[1])
        if ws is None or ws.numel() < need:
            ws = self._pool_ws = torch.empty(need, dtype=torch.uint8, device=dev)
        return B.pkv_append_and_decode_pools(pools, k_new, v_new, self._sl_dev[:n], q, self._sl_dev[n:2 * n], scale,
                                             out=out, workspace=ws)
