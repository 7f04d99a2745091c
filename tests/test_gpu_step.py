"""The one-call decode step (pkv_decode_step_host via
PagedKVCache.decode_step_host) against the multi-call step and the oracle:
the same allocator operations, the same pool bytes and the same outputs, with
copy-on-write pairs (forked sequences) in the step, for 16-bit and e4m3 pools."""
import numpy as np
import pytest
import torch

from helpers import DT, assert_close, raw
from oracle import paged_attention as pa
from oracle.block_allocator import BlockAllocatorModel

pytestmark = pytest.mark.gpu

import paged_kv_cache_406_b200 as pkv  # noqa: E402
from paged_kv_cache_406_b200.cache import PagedKVCache  # noqa: E402


def _caches(dtype, nb=64, hkv=2, d=128, bs=16, seed=3):
    rng = np.random.default_rng(seed)
    order = rng.permutation(nb)
    shape = (nb, hkv, bs, d)
    if dtype == "e4m3":
        codes = torch.from_numpy(rng.integers(0, 0x7F, size=shape, dtype=np.uint8))  # finite codes
        kp, vp = codes.clone(), codes.flip(0).clone()
        tdt = torch.uint8
    else:
        kp = torch.from_numpy(rng.standard_normal(shape, dtype=np.float32)).to(DT[dtype])
        vp = torch.from_numpy(rng.standard_normal(shape, dtype=np.float32)).to(DT[dtype])
        tdt = DT[dtype]
    mk = lambda: PagedKVCache(nb, hkv, d, bs, tdt, 16, device="cuda", free_order=order,  # noqa: E731
                              k_pool=kp.clone().cuda(), v_pool=vp.clone().cuda(), k_scale=0.5, v_scale=0.25)
    return mk(), mk(), order, kp, vp


@pytest.mark.parametrize("dtype", ["bf16", "f16", "e4m3"])
def test_one_call_step_matches_multi_call_step_and_oracle(native, dtype):
    pkv.pkv_device_status(clear=True)
    a, b, order, kp0, vp0 = _caches(dtype)
    lens = [5, 16, 40, 1]
    model = BlockAllocatorModel(64, 16, order)
    for c in (a, b):
        for i, L in enumerate(lens):
            c.add(i, L)
        c.fork(2, 4)  # sequence 4 shares sequence 2's partial last block: one copy-on-write pair
    for i, L in enumerate(lens):
        model.add(i, L)
    model.fork(2, 4)
    ids = np.array([0, 1, 2, 3, 4], dtype=np.int64)
    rng = np.random.default_rng(9)
    io = torch.float16 if dtype == "e4m3" else DT[dtype]
    q = torch.from_numpy(rng.standard_normal((5, 8, 128), dtype=np.float32)).to(io)
    kn = torch.from_numpy(rng.standard_normal((5, 2, 128), dtype=np.float32)).to(io)
    vn = torch.from_numpy(rng.standard_normal((5, 2, 128), dtype=np.float32)).to(io)
    scale = 1 / np.sqrt(128)
    ref_out = a.decode_step(list(ids), q.cuda(), kn.cuda(), vn.cuda(), scale).clone()
    out_host = torch.empty((5, 8, 128), dtype=torch.float32, pin_memory=True)
    pinned = (q.pin_memory(), kn.pin_memory(), vn.pin_memory())
    got = b.decode_step_host(ids, *pinned, scale, out_host=out_host)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(clear=True) == 0
    assert torch.equal(got, ref_out.cpu()), "one-call and multi-call steps differ"
    assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool)
    assert a.stats() == b.stats() and a.stats()["cow_copies"] == 1
    if dtype == "e4m3":
        return  # the e4m3 step itself is checked against the oracle in test_gpu_fp8.py
    slots, cows = model.append_slots(list(ids))
    kc, vc = pa.copy_blocks(raw(kp0), raw(vp0), cows)
    ek, ev = pa.kv_append(kc, vc, raw(kn), raw(vn), np.array(slots))
    assert np.array_equal(raw(b.k_pool), ek) and np.array_equal(raw(b.v_pool), ev)
    tables = np.full((5, 16), -1, dtype=np.int32)
    for i in range(5):
        t = model.block_table(i)
        tables[i, :len(t)] = t
    ref = pa.paged_decode_attention(raw(q), ek, ev, tables, np.array([model.seq_len(i) for i in range(5)]), scale,
                                    dtype)
    assert_close(got, ref, dtype, f"one-call step {dtype}")


def test_one_call_steps_in_a_row(native):
    """Twenty steps, with and without the copy streams: the two buffer sets
    alternate safely."""
    a, b, order, _, _ = _caches("bf16", nb=128)
    for c in (a, b):
        for i in range(6):
            c.add(i, 3 * i + 1)
    ids = np.arange(6, dtype=np.int64)
    rng = np.random.default_rng(1)
    for step in range(20):
        q = torch.from_numpy(rng.standard_normal((6, 8, 128), dtype=np.float32)).to(torch.bfloat16)
        kn = torch.from_numpy(rng.standard_normal((6, 2, 128), dtype=np.float32)).to(torch.bfloat16)
        vn = torch.from_numpy(rng.standard_normal((6, 2, 128), dtype=np.float32)).to(torch.bfloat16)
        r = a.decode_step(list(ids), q.cuda(), kn.cuda(), vn.cuda(), 0.1).clone()
        pinned = (q.pin_memory(), kn.pin_memory(), vn.pin_memory())  # alive until the copies have run
        g = b.decode_step_host(ids, *pinned, 0.1, overlap=step % 2 == 0)
        assert torch.equal(r, g), f"step {step}"
        torch.cuda.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(a.k_pool, b.k_pool)
    assert pkv.pkv_device_status(clear=True) == 0


def test_one_call_steps_with_changing_batches(native):
    """The batch size and the partition size change from step to step (as a
    serving loop's do): the one-call step reuses its buffers for smaller
    batches, grows them for larger ones, re-derives its call arguments, and
    matches the multi-call step bit for bit, with and without the copy
    streams."""
    a, b, _, _, _ = _caches("bf16", nb=128)
    for c in (a, b):
        for i in range(6):
            c.add(i, 5 * i + 2)
    rng = np.random.default_rng(7)
    for step, n in enumerate([3, 1, 6, 2, 6, 4, 1, 5, 6, 3, 2, 6]):
        ids = np.arange(n, dtype=np.int64)
        pt = (0, 32, 64)[step % 3]
        q = torch.from_numpy(rng.standard_normal((n, 8, 128), dtype=np.float32)).to(torch.bfloat16)
        kn = torch.from_numpy(rng.standard_normal((n, 2, 128), dtype=np.float32)).to(torch.bfloat16)
        vn = torch.from_numpy(rng.standard_normal((n, 2, 128), dtype=np.float32)).to(torch.bfloat16)
        r = a.decode_step(list(ids), q.cuda(), kn.cuda(), vn.cuda(), 0.1, partition_tokens=pt).clone()
        pinned = (q.pin_memory(), kn.pin_memory(), vn.pin_memory())  # alive until the copies have run
        out_host = torch.empty((n, 8, 128), dtype=torch.float32, pin_memory=True)
        g = b.decode_step_host(ids, *pinned, 0.1, out_host=out_host, partition_tokens=pt, overlap=step % 4 != 3)
        b.wait_copies()
        torch.cuda.synchronize()
        assert torch.equal(r.cpu(), g), f"step {step} (n {n}, partitions of {pt})"
    torch.cuda.synchronize()
    assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool)
    assert pkv.pkv_device_status(clear=True) == 0
