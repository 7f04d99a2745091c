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
@pytest.mark.parametrize("one_call", [True, False])
def test_adaptive_decode_step_matches_oracle(native, one_call):
    """All classes in one pkv_append_and_decode_pools call, and one call per
    class; both against the oracle."""
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
    out = cache.decode_step(ids, q.pin_memory(), kn.pin_memory(), vn.pin_memory(), scale, one_call=one_call)
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
        assert np.array_equal(raw(cache.caches[bs].k_pool), kp), f"class bs{bs}: K pool"
        assert np.array_equal(raw(cache.caches[bs].v_pool), vp), f"class bs{bs}: V pool"
        ref = pa.paged_decode_attention(raw(q[a:a + m]), kp, vp, tables,
                                        np.array([models[bs].seq_len(s) for s in members]), scale, dtype)
        assert_close(out[a:a + m], ref, dtype, f"class bs{bs}")
        a += m


@pytest.mark.gpu
@pytest.mark.parametrize("lens,g,dtype", [
    ([5, 700, 9000, 8192, 20000], 4, "bf16"),   # no 16-token class: the middle pool is empty
    ([1024, 3000, 4096, 100], 8, "f16"),        # no 8-token class
    ([9000], 2, "bf16"),                        # one class only
])
def test_pools_call_with_missing_classes(native, lens, g, dtype):
    """pkv_append_and_decode_pools with classes that hold no sequence, three
    steps in a row (a step crossing block boundaries); pools byte for byte
    and attention against the oracle at the last step."""
    pkv.pkv_device_status(clear=True)
    rng = np.random.default_rng(len(lens) * 7 + g)
    hkv, d = 2, 128
    hq = g * hkv
    steps = 3
    per_class = {32: 0, 16: 0, 8: 0}
    for L in lens:
        per_class[block_size_for(L)] += -(-(L + steps) // block_size_for(L)) + 1
    per_class = {bs: max(nb, 1) for bs, nb in per_class.items()}  # every class gets a pool, some stay unused
    cache = AdaptivePagedKVCache(per_class, hkv, d, DT[dtype], max_tokens=max(lens) + steps, seed=9)
    models, pools0 = {}, {}
    for bs, c in cache.caches.items():
        models[bs] = BlockAllocatorModel(c.num_blocks, bs,
                                         np.random.Generator(np.random.PCG64(9 + bs)).permutation(c.num_blocks))
        c.k_pool.copy_(torch.from_numpy(rng.standard_normal(c.k_pool.shape, dtype=np.float32)).to(DT[dtype]))
        c.v_pool.copy_(torch.from_numpy(rng.standard_normal(c.v_pool.shape, dtype=np.float32)).to(DT[dtype]))
        pools0[bs] = [raw(c.k_pool), raw(c.v_pool)]
    for i, L in enumerate(lens):
        models[cache.add(i, L)].add(i, L)
    ids = cache.order()
    n = len(ids)
    scale = 1.0 / np.sqrt(d)
    for step in range(steps):
        q = torch.from_numpy(rng.standard_normal((n, hq, d), dtype=np.float32)).to(DT[dtype])
        kn = torch.from_numpy(rng.standard_normal((n, hkv, d), dtype=np.float32)).to(DT[dtype])
        vn = torch.from_numpy(rng.standard_normal((n, hkv, d), dtype=np.float32)).to(DT[dtype])
        out = cache.decode_step(ids, q, kn, vn, scale)
        torch.cuda.synchronize()
        assert pkv.pkv_device_status(clear=True) == 0
        a = 0
        for bs in (32, 16, 8):
            members = [i for i in ids if cache.cls[i] == bs]
            if not members:
                continue
            m = len(members)
            slots, _ = models[bs].append_slots(members)
            pools0[bs] = list(pa.kv_append(*pools0[bs], raw(kn[a:a + m]), raw(vn[a:a + m]), np.array(slots)))
            a += m
    a = 0
    for bs in (32, 16, 8):
        members = [i for i in ids if cache.cls[i] == bs]
        if not members:
            continue
        m = len(members)
        kp, vp = pools0[bs]
        assert np.array_equal(raw(cache.caches[bs].k_pool), kp), f"class bs{bs}: K pool"
        assert np.array_equal(raw(cache.caches[bs].v_pool), vp), f"class bs{bs}: V pool"
        maxb = max(len(models[bs].block_table(x)) for x in members)
        tables = np.full((m, maxb), -1, dtype=np.int32)
        for r, x in enumerate(members):
            t = models[bs].block_table(x)
            tables[r, :len(t)] = t
        ref = pa.paged_decode_attention(raw(q[a:a + m]), kp, vp, tables,
                                        np.array([models[bs].seq_len(x) for x in members]), scale, dtype)
        assert_close(out[a:a + m], ref, dtype, f"class bs{bs} after {steps} steps")
        a += m


@pytest.mark.gpu
def test_pools_call_refuses_bad_pool_lists(native):
    dev = "cuda"
    kp = torch.zeros((4, 1, 16, 128), dtype=torch.bfloat16, device=dev)
    t = torch.zeros((1, 1), dtype=torch.int32, device=dev)
    one = torch.ones(1, dtype=torch.int32, device=dev)
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device=dev)
    kn = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device=dev)
    with pytest.raises(pkv.PagedKVError) as e:  # four pools: at most three
        pkv.pkv_append_and_decode_pools([(kp, kp, t, 0)] * 3 + [(kp, kp, t, 1)], kn, kn, one, q, one, 0.1)
    assert e.value.code == -1
    with pytest.raises(pkv.PagedKVError) as e:  # partition not a multiple of the 32-token block size
        kp32 = torch.zeros((4, 1, 32, 128), dtype=torch.bfloat16, device=dev)
        pkv.pkv_append_and_decode_pools([(kp32, kp32, t, 1)], kn, kn, one, q, one, 0.1, partition_tokens=48)
    assert e.value.code == -1
    with pytest.raises(pkv.PagedKVError) as e:  # one query head per KV head: not a tensor-core group
        pkv.pkv_append_and_decode_pools([(kp, kp, t, 1)], kn, kn, one, q[:, :1], one, 0.1)
    assert e.value.code == -4
    assert pkv.pkv_device_status(clear=True) == 0
