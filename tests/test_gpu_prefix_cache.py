"""Prefix caching end to end on the GPU: a request admitted with
add_cached reuses the K/V blocks an earlier request with the same prefix
left cached; only its new tokens are appended and prefilled; its attention
over the whole prompt (cached prefix + new tokens) and the next decode step
match the oracle run on the request's full K/V (vLLM paging page §3 phase 3,
production page §5)."""
import numpy as np
import pytest
import torch

from helpers import assert_close, raw
from oracle import paged_attention as pa

pytestmark = pytest.mark.gpu

import paged_kv_cache_406_b200 as pkv  # noqa: E402
from paged_kv_cache_406_b200.cache import PagedKVCache  # noqa: E402

BS, HKV, HQ, D = 16, 2, 8, 128


def _slots(cache, sid, start, end):
    tables, _ = cache.alloc.block_tables([sid], cache.max_blocks)
    t = np.arange(start, end)
    return (tables[0, t // BS] * BS + t % BS).astype(np.int32)


def _prefill(cache, sid, q, k, v, start, end, scale):
    """Append rows start..end-1 of the prompt and run its prefill chunk."""
    slots = torch.from_numpy(_slots(cache, sid, start, end)).cuda()
    pkv.pkv_kv_append(k[start:end].cuda(), v[start:end].cuda(), slots, cache.k_pool, cache.v_pool)
    tables, lens = cache.alloc.block_tables([sid], cache.max_blocks)
    n = end - start
    return pkv.pkv_paged_attention_prefill(q.cuda(), cache.k_pool, cache.v_pool, torch.from_numpy(tables).cuda(),
                                           torch.from_numpy(lens).cuda(),
                                           torch.tensor([0, n], dtype=torch.int32, device="cuda"), n, scale)


def test_cached_prefix_prefill_and_decode(native):
    pkv.pkv_device_status(clear=True)
    rng = np.random.default_rng(11)
    nb = 64
    cache = PagedKVCache(nb, HKV, D, BS, torch.bfloat16, 16, device="cuda", free_order=rng.permutation(nb))
    cache.k_pool.zero_()
    cache.v_pool.zero_()
    scale = 1 / np.sqrt(D)
    randn = lambda *s: torch.from_numpy(rng.standard_normal(s, dtype=np.float32)).to(torch.bfloat16)  # noqa: E731

    # request A: 100 prompt tokens, nothing cached yet
    toks_a = rng.integers(0, 32000, size=100)
    ka, va = randn(100, HKV, D), randn(100, HKV, D)
    assert cache.add_cached(0, toks_a) == 0
    _prefill(cache, 0, randn(100, HQ, D), ka, va, 0, 100, scale)
    torch.cuda.synchronize()
    blocks_a = cache.alloc.block_tables([0], 16)[0][0, :7].tolist()
    cache.free(0)  # A ends: its 6 full blocks stay cached

    # request B: A's first 64 tokens, then 50 of its own
    toks_b = np.concatenate([toks_a[:64], rng.integers(0, 32000, size=50)])
    assert cache.add_cached(1, toks_b) == 64
    tab_b = cache.alloc.block_tables([1], 16)[0][0]
    assert tab_b[:4].tolist() == blocks_a[:4]  # the cached blocks are reused, not copied
    kb = torch.cat([ka[:64], randn(50, HKV, D)])
    vb = torch.cat([va[:64], randn(50, HKV, D)])
    qb = randn(50, HQ, D)
    out = _prefill(cache, 1, qb, kb, vb, 64, 114, scale)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(clear=True) == 0

    # oracle on B's full K/V, in a pool of its own (no shared state)
    nbb = -(-114 // BS)
    kp = np.zeros((nbb, HKV, BS, D), dtype=np.uint16)
    vp = np.zeros_like(kp)
    t = np.arange(114)
    kp[t // BS, :, t % BS] = raw(kb)
    vp[t // BS, :, t % BS] = raw(vb)
    ref = pa.paged_prefill_attention(raw(qb), kp, vp, np.arange(nbb)[None], np.array([114]), np.array([50]), scale,
                                     "bf16")
    assert_close(out, ref, "bf16", "prefill over the cached prefix")

    # one decode step of B on top
    qd, kd, vd = randn(1, HQ, D), randn(1, HKV, D), randn(1, HKV, D)
    dec = cache.decode_step([1], qd.cuda(), kd.cuda(), vd.cuda(), scale)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(clear=True) == 0
    kp2 = np.zeros((-(-115 // BS), HKV, BS, D), dtype=np.uint16)
    vp2 = np.zeros_like(kp2)
    t = np.arange(115)
    kp2[t // BS, :, t % BS] = np.concatenate([raw(kb), raw(kd)])
    vp2[t // BS, :, t % BS] = np.concatenate([raw(vb), raw(vd)])
    ref2 = pa.paged_decode_attention(raw(qd), kp2, vp2, np.arange(kp2.shape[0])[None], np.array([115]), scale, "bf16")
    assert_close(dec, ref2, "bf16", "decode after the cached prefix")
    st = cache.stats()
    assert st["cache_hits"] == 4 and st["cache_queries"] == 6 + 7
