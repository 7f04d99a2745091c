"""Adaptive block size (optimisation-overview page §3.3): sequences routed to
pools of 32-, 16- or 8-token blocks by length; one decode step through
AdaptivePagedKVCache against the fp64 oracle (expected slots and tables from
the oracle's allocator model, append and attention from the oracle)."""
import numpy as np
import pytest
import torch

from helpers import DT, assert_close, raw
from oracle import paged_attention as pa
from oracle.block_allocator import BlockAllocatorModel

import paged_kv_cache_406_b200 as pkv  # noqa: E402
from paged_kv_cache_406_b200.cache import AdaptivePagedKVCache, block_size_for  # noqa: E402


def test_block_size_classes():
    assert [block_size_for(n) for n in (0, 1, 1023, 1024, 8191, 8192, 100000)] == [32, 32, 32, 16, 16, 8, 8]


@pytest.mark.gpu
def test_adaptive_decode_step_matches_oracle(native):
    pkv.pkv_device_status(clear=True)
    rng = np.random.default_rng(33)
    hq, hkv, d, dtype = 8, 2, 128, "bf16"
    lens = [5, 1023, 1024, 3000, 8191, 8192, 9000, 100, 32, 700]
    per_class = {32: 0, 16: 0, 8: 0}
    for L in lens:
        bs = block_size_for(L)
        per_class[bs] += -(-(L + 1) // bs) + 1
    cache = AdaptivePagedKVCache(per_class, hkv, d, DT[dtype], max_tokens=9100, seed=5)
    models = {}
    for bs, c in cache.caches.items():
        order = np.random.Generator(np.random.PCG64(5 + bs)).permutation(c.num_blocks)
        models[bs] = BlockAllocatorModel(c.num_blocks, bs, order)
        c.k_pool.copy_(torch.from_numpy(rng.standard_normal(c.k_pool.shape, dtype=np.float32)).to(DT[dtype]))
        c.v_pool.copy_(torch.from_numpy(rng.standard_normal(c.v_pool.shape, dtype=np.float32)).to(DT[dtype]))
    pools0 = {bs: (raw(c.k_pool), raw(c.v_pool)) for bs, c in cache.caches.items()}
    for i, L in enumerate(lens):
        bs = cache.add(i, L)
        models[bs].add(i, L)
    ids = cache.order()
    assert [block_size_for(lens[i]) for i in ids] == sorted((block_size_for(lens[i]) for i in ids), reverse=True)
    n = len(ids)
    q = torch.from_numpy(rng.standard_normal((n, hq, d), dtype=np.float32)).to(DT[dtype])
    kn = torch.from_numpy(rng.standard_normal((n, hkv, d), dtype=np.float32)).to(DT[dtype])
    vn = torch.from_numpy(rng.standard_normal((n, hkv, d), dtype=np.float32)).to(DT[dtype])
    scale = 1.0 / np.sqrt(d)
    out = cache.decode_step(ids, q.pin_memory(), kn.pin_memory(), vn.pin_memory(), scale)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(clear=True) == 0

    a = 0
    for bs in (32, 16, 8):
        members = [i for i in ids if block_size_for(lens[i]) == bs]
        if not members:
            continue
        m = len(members)
        slots, _ = models[bs].append_slots(members)
        kp, vp = pa.kv_append(*pools0[bs], raw(kn[a:a + m]), raw(vn[a:a + m]), np.array(slots))
        maxb = max(len(models[bs].block_table(s)) for s in members)
        tables = np.full((m, maxb), -1, dtype=np.int32)
        for r, s in enumerate(members):
            t = models[bs].block_table(s)
            tables[r, :len(t)] = t
        ref = pa.paged_decode_attention(raw(q[a:a + m]), kp, vp, tables,
                                        np.array([models[bs].seq_len(s) for s in members]), scale, dtype)
        assert_close(out[a:a + m], ref, dtype, f"class bs{bs}")
        a += m
