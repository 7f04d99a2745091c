"""Runs a seeded workload through the library (PagedKVCache) and mirrors every
step on the oracle side for a sample of sequences.

The oracle side never reads a value the CUDA path produced: its pool blocks
come from the pristine initial pool (torch's seeded generator), its slots and
tables from the oracle's own allocator model, and its appended rows from the
step's seeded inputs.  GPU results are compared after each checked step.
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


class Mirror:
    """Host copies of the blocks the sampled sequences use (compact ids)."""

    def __init__(self, k0: torch.Tensor, v0: torch.Tensor):
        self.k0, self.v0 = k0, v0
        self.ids: dict[int, int] = {}
        self.k: list[np.ndarray] = []
        self.v: list[np.ndarray] = []

    def block(self, phys: int) -> int:
        if phys not in self.ids:
            self.ids[phys] = len(self.k)
            self.k.append(raw(self.k0[phys]).copy())
            self.v.append(raw(self.v0[phys]).copy())
        return self.ids[phys]

    def append(self, slot: int, krow: np.ndarray, vrow: np.ndarray, bs: int) -> None:
        blk, off = divmod(int(slot), bs)
        c = self.block(blk)
        self.k[c][:, off, :] = krow
        self.v[c][:, off, :] = vrow

    def copy(self, src: int, dst: int) -> None:
        s, d = self.block(src), self.block(dst)
        self.k[d] = self.k[s].copy()
        self.v[d] = self.v[s].copy()



def run_workload(w: W.Workload, sample, check, steps=None, prefix_tokens=None, heads=None):
    """Runs ``steps`` decode steps of ``w``; after each step, for every sampled
    sequence b with ``check(step, b)`` true, compares its blocks byte for byte
    and its attention output (KV heads ``heads``, all if None) with the oracle.
    ``sample``: sequence indices mirrored on the host (None = all).
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
    model = BlockAllocatorModel(nb, bs, order)
    B = w.num_seqs
    sample = set(range(B)) if sample is None else set(sample)
    mirror = Mirror(k0, v0)
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
                for s_, d_ in mcow:
                    mirror.copy(s_, d_)
            pkv_kv_append(kn.cuda(), vn.cuda(), dslots, cache.k_pool, cache.v_pool)
            kr, vr = raw(kn), raw(vn)
            for i, b in enumerate(ids):
                if b in sample:
                    mirror.append(mslots[i], kr[i], vr[i], bs)
    else:
        for b in range(B):
            cache.add(b, int(lens[b]))
            model.add(b, int(lens[b]))

    for step in range(steps):
        ids = list(range(B))
        mslots, mcow = model.append_slots(ids)
        for s_, d_ in mcow:
            mirror.copy(s_, d_)
        q = W.normal((B, hq, d), dt, W.step_seed(w, step, 0))
        kn = W.normal((B, hkv, d), dt, W.step_seed(w, step, 1))
        vn = W.normal((B, hkv, d), dt, W.step_seed(w, step, 2))
        out = cache.decode_step(ids, q, kn, vn, w.scale, partition_tokens=w.partition_tokens)
        torch.cuda.synchronize()
        gslots = cache._meta_dev[:B].cpu().numpy()
        assert gslots.tolist() == mslots, f"step {step}: slot mapping differs from the allocator model"
        kr, vr, qr = raw(kn), raw(vn), raw(q)
        for b in sample:
            mirror.append(mslots[b], kr[b], vr[b], bs)
        for b in sorted(sample):
            if not check(step, b):
                continue
            tab = model.block_table(b)
            L = model.seq_len(b)
            ks = np.stack([mirror.k[mirror.block(p)] for p in tab])
            vs = np.stack([mirror.v[mirror.block(p)] for p in tab])
            idx = torch.tensor(tab, device="cuda")
            assert np.array_equal(raw(cache.k_pool[idx]), ks), f"K blocks of seq {b} differ at step {step}"
            assert np.array_equal(raw(cache.v_pool[idx]), vs), f"V blocks of seq {b} differ at step {step}"
            local = np.arange(len(tab), dtype=np.int32)[None]
            for g in (range(hkv) if heads is None else heads):
                ref = pa.paged_decode_attention(qr[b:b + 1, g * G:(g + 1) * G], ks[:, g:g + 1], vs[:, g:g + 1],
                                                local, np.array([L]), w.scale, w.dtype)
                assert_close(out[b:b + 1, g * G:(g + 1) * G], ref, w.dtype,
                             f"{w.name} step {step} seq {b} kv head {g}")
    assert pkv_device_status(clear=True) == 0
    return cache.stats()
