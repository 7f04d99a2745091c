"""Runs a seeded workload through the library (PagedKVCache) and mirrors every
step on the oracle side.

The oracle side never reads a value the CUDA path produced: its pool starts as
a host copy of the pristine initial pool (torch's seeded generator), its slots,
tables and copy-on-write pairs come from the oracle's own allocator model, and
its appended rows from the step's seeded inputs.  The host pool is kept up to
date for every sequence (copy-on-write copies and appends applied in place, as
the oracle's ``copy_blocks`` and ``kv_append`` define them), so any checked
sequence can be compared at any step.
"""
from __future__ import annotations

import numpy as np
import torch

from helpers import assert_close, raw
from oracle import paged_attention as pa
from oracle.block_allocator import BlockAllocatorModel
from paged_kv_cache_406_b200 import pkv_copy_blocks, pkv_device_status, pkv_kv_append
from paged_kv_cache_406_b200 import workloads as W
from paged_kv_cache_406_b200.cache import PagedKVCache


class HostPool:
    """The oracle's copy of both pools, raw storage, updated in place."""

    def __init__(self, k0: torch.Tensor, v0: torch.Tensor, bs: int):
        self.k, self.v, self.bs = raw(k0).copy(), raw(v0).copy(), bs

    def copy(self, pairs) -> None:
        # copy_blocks: whole blocks src -> dst, in order
        for src, dst in pairs:
            self.k[dst] = self.k[src]
            self.v[dst] = self.v[src]

    def append(self, slots, krows: np.ndarray, vrows: np.ndarray) -> None:
        # kv_append: row i into block slot // bs at offset slot % bs; slot < 0 writes nothing
        for i, s in enumerate(slots):
            if s < 0:
                continue
            blk, off = divmod(int(s), self.bs)
            self.k[blk, :, off, :] = krows[i]
            self.v[blk, :, off, :] = vrows[i]


def compare_pools(cache: PagedKVCache, host: HostPool, what: str) -> None:
    """Every byte of both device pools against the oracle's host pools."""
    assert np.array_equal(raw(cache.k_pool), host.k), f"{what}: K pool differs from the oracle's"
    assert np.array_equal(raw(cache.v_pool), host.v), f"{what}: V pool differs from the oracle's"


def run_workload(w: W.Workload, sample, check, steps=None, prefix_tokens=None, heads=None):
    """Runs ``steps`` decode steps of ``w``.  After each step the slot
    mapping is compared with the allocator model's, and for every sequence b
    in ``sample`` (None = all) with ``check(step, b)`` true the attention
    output (KV heads ``heads``, None = all) is compared with the fp64 oracle.
    Both pools are compared byte for byte in full after the prefix phase,
    after the first step and after the last one (pools only grow, so a wrong
    write at any step is still there at the end).
    Returns the allocator stats after the last step."""
    steps = w.steps if steps is None else steps
    dt = w.torch_dtype
    bs, hkv, d, hq, G = w.block_size, w.num_kv_heads, w.head_dim, w.num_q_heads, w.group
    lens = W.seq_lens(w)
    prefix = w.prefix_tokens if prefix_tokens is None else prefix_tokens
    if w.prefix_tokens:
        lens = lens - w.prefix_tokens + prefix
    nb = W.pool_blocks(w, lens) + (w.num_seqs if prefix else 0)
    order = W.free_order(nb, w.seed)
    shape = (nb, hkv, bs, d)
    k0 = W.normal(shape, dt, W.pool_seed(w, 0), device="cuda")
    v0 = W.normal(shape, dt, W.pool_seed(w, 1), device="cuda")
    maxb = -(-(int(lens.max()) + steps) // bs)
    cache = PagedKVCache(nb, hkv, d, bs, dt, maxb, free_order=order, k_pool=k0.clone(), v_pool=v0.clone())
    host = HostPool(k0, v0, bs)
    del k0, v0
    model = BlockAllocatorModel(nb, bs, order)
    B = w.num_seqs
    sample = set(range(B)) if sample is None else set(sample)
    rng = np.random.default_rng(w.seed + 77)

    # ---- admit the batch (shared prefix: one sequence, forked, then tails) ----
    if prefix:
        cache.add(0, prefix)
        model.add(0, prefix)
        for b in range(1, B):
            cache.fork(0, b)
            model.fork(0, b)
        tails = lens - prefix
        for r in range(int(tails.max())):
            ids = [b for b in range(B) if tails[b] > r]
            ncow, (slots, _, cow, _) = cache.prepare_step(ids)
            mslots, mcow = model.append_slots(ids)
            assert slots[:len(ids)].tolist() == mslots
            assert [tuple(x) for x in cow[:2 * ncow].reshape(-1, 2).tolist()] == mcow
            dslots, _, dcow, _ = cache.upload_step(len(ids))
            kn = W.normal((len(ids), hkv, d), dt, int(rng.integers(1 << 30)))
            vn = W.normal((len(ids), hkv, d), dt, int(rng.integers(1 << 30)))
            if ncow:
                pkv_copy_blocks(cache.k_pool, cache.v_pool, dcow[:2 * ncow].view(ncow, 2))
                host.copy(mcow)
            pkv_kv_append(kn.cuda(), vn.cuda(), dslots, cache.k_pool, cache.v_pool)
            host.append(mslots, raw(kn), raw(vn))
        torch.cuda.synchronize()
        compare_pools(cache, host, f"{w.name} after the prefix phase")
    else:
        for b in range(B):
            cache.add(b, int(lens[b]))
            model.add(b, int(lens[b]))

    for step in range(steps):
        ids = list(range(B))
        mslots, mcow = model.append_slots(ids)
        host.copy(mcow)
        q = W.normal((B, hq, d), dt, W.step_seed(w, step, 0))
        kn = W.normal((B, hkv, d), dt, W.step_seed(w, step, 1))
        vn = W.normal((B, hkv, d), dt, W.step_seed(w, step, 2))
        out = cache.decode_step(ids, q, kn, vn, w.scale, partition_tokens=w.partition_tokens)
        torch.cuda.synchronize()
        gslots = cache._meta_dev[:B].cpu().numpy()
        assert gslots.tolist() == mslots, f"step {step}: slot mapping differs from the allocator model"
        qr = raw(q)
        host.append(mslots, raw(kn), raw(vn))
        if step in (0, steps - 1):
            compare_pools(cache, host, f"{w.name} step {step}")
        out_h = out.cpu()
        for b in sorted(sample):
            if not check(step, b):
                continue
            tab = np.asarray(model.block_table(b))
            L = model.seq_len(b)
            local = np.arange(len(tab), dtype=np.int32)[None]
            ks, vs = host.k[tab], host.v[tab]
            for g in (range(hkv) if heads is None else heads):
                ref = pa.paged_decode_attention(qr[b:b + 1, g * G:(g + 1) * G], ks[:, g:g + 1], vs[:, g:g + 1],
                                                local, np.array([L]), w.scale, w.dtype)
                assert_close(out_h[b:b + 1, g * G:(g + 1) * G], ref, w.dtype,
                             f"{w.name} step {step} seq {b} kv head {g}")
    assert pkv_device_status(clear=True) == 0
    return cache.stats()
