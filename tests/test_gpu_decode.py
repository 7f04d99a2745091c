"""GPU parity: append, block copy and paged decode attention through the
C-ABI against the fp64 oracle, on seeded inputs (B200).

Tolerance: |gpu - oracle| <= tol * max(1, |oracle|) elementwise, tol = 1e-5 for
fp32 K/V and 2e-3 for bf16 / fp16 K/V (fp32 output).  Append and copy are
compared byte for byte over the whole pool.
"""
import zlib

import numpy as np
import pytest
import torch

from helpers import DT, TOL, Case, assert_close, randn, raw
from oracle import paged_attention as pa
from oracle.block_allocator import BlockAllocatorModel

pytestmark = pytest.mark.gpu

import paged_kv_cache_406_b200 as pkv  # noqa: E402


@pytest.fixture(autouse=True)
def _clean_status(native):
    pkv.pkv_device_status(clear=True)
    yield
    assert pkv.pkv_device_status(clear=True) == 0, "a kernel recorded a device error"


def _decode(case: Case, pt=0, lens=None):
    d = case.device()
    if lens is not None:
        d["seq_lens"] = torch.from_numpy(np.asarray(lens, dtype=np.int32)).cuda()
    out = pkv.pkv_paged_attention_decode(d["q"], d["k_pool"], d["v_pool"], d["block_tables"], d["seq_lens"],
                                         case.scale, partition_tokens=pt)
    torch.cuda.synchronize()
    return out


def _ragged(bs):
    return [0, 1, bs - 1, bs, bs + 1, 2 * bs + 3, 100, 255, 256, 257, 511, 512, 513, 1025]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_decode_matches_oracle(dtype, d, g, bs):
    """16-bit K/V with G >= 2 runs on the tensor-core kernel, the rest on the
    CUDA-core kernel; both against the oracle on ragged lengths."""
    if dtype == "f32" and g == 8:
        pytest.skip("group size 8 needs 16-bit K/V (rejected: see test_unsupported_group)")
    hkv = 2
    case = Case(_ragged(bs), g * hkv, hkv, d, bs, dtype, seed=zlib.crc32(f"{dtype}{d}{g}{bs}".encode()) % 1000)
    ref = case.oracle()
    out = _decode(case)  # automatic 512-token partitions: the 513- and 1025-token sequences are split
    assert_close(out, ref, dtype, f"{dtype} D{d} G{g} bs{bs}")


@pytest.mark.parametrize("pt_blocks", [1, 2, 5, 64])
def test_partition_sizes_agree(pt_blocks):
    bs = 16
    case = Case([1, 15, 16, 17, 160, 333, 1000, 1024, 1025], 8, 2, 128, bs, "bf16", seed=11)
    ref = case.oracle()
    out = _decode(case, pt=bs * pt_blocks)
    assert_close(out, ref, "bf16", f"partition {bs * pt_blocks}")
    single = _decode(case, pt=8192)
    assert torch.max(torch.abs(out - single)).item() < 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("g", [2, 4, 8])
def test_tensor_core_and_cuda_core_kernels_agree(dtype, g):
    """partition_tokens 24 (not a multiple of 16) sends 16-bit GQA work to the
    CUDA-core kernel; 32 to the tensor-core kernel.  Both match the oracle."""
    if g == 8:
        pytest.skip("the CUDA-core kernel covers group sizes 1, 2, 4")
    case = Case([1, 7, 8, 9, 23, 24, 25, 200, 777], 2 * g, 2, 128, 8, dtype, seed=21)
    ref = case.oracle()
    simt = _decode(case, pt=24)
    mma = _decode(case, pt=32)
    assert_close(simt, ref, dtype, "cuda-core kernel")
    assert_close(mma, ref, dtype, "tensor-core kernel")
    assert torch.max(torch.abs(simt - mma)).item() < 2e-3


def test_unsupported_group():
    case = Case([5], 8, 1, 64, 16, "f32", seed=22)
    with pytest.raises(pkv.PagedKVError) as e:
        _decode(case)
    assert e.value.code == pkv._native.PKV_ERR_UNSUPPORTED


def test_softmax_peaked_two_tokens_meets_tolerance():
    """Two tokens with scores far apart and large V: the hi + lo split of P
    keeps the weighted sum within tolerance where a single 16-bit P would not."""
    case = Case([2, 3, 2], 8, 2, 128, 16, "bf16", seed=23)
    case.v_pool.mul_(8.0)
    case.q.mul_(3.0)
    ref = case.oracle()
    assert_close(_decode(case), ref, "bf16", "peaked")


def test_zero_length_gives_zeros_and_single_token_gives_v():
    case = Case([0, 1, 0, 1], 4, 1, 128, 16, "bf16", seed=3)
    out = _decode(case)
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0
    for b in (1, 3):
        blk = case.tables[b, 0]
        v = case.v_pool[blk, 0, 0].float().cuda()
        for h in range(4):
            assert torch.equal(out[b, h], v), "seq_len 1 must return v exactly"


def test_constant_v_gives_constant():
    case = Case([5, 300, 2000], 8, 2, 128, 16, "f16", seed=4)
    case.v_pool.fill_(1.0)
    out = _decode(case)
    assert torch.max(torch.abs(out - 1.0)).item() < 1e-6


def test_bit_identical_under_block_permutation():
    lens = [3, 77, 600, 1300]
    a = Case(lens, 8, 2, 128, 16, "bf16", seed=5)
    b = Case(lens, 8, 2, 128, 16, "bf16", seed=6)
    # give b the same logical contents as a, at b's physical blocks
    for s, L in enumerate(lens):
        for j in range(-(-L // 16)):
            b.k_pool[b.tables[s, j]] = a.k_pool[a.tables[s, j]]
            b.v_pool[b.tables[s, j]] = a.v_pool[a.tables[s, j]]
    b.q = a.q.clone()
    oa, ob = _decode(a), _decode(b)
    assert torch.equal(oa, ob)
    oa2 = _decode(a)
    assert torch.equal(oa, oa2), "decode must be deterministic"


def test_attention_uses_contiguous_gqa_groups():
    case = Case([40, 40], 8, 2, 64, 16, "f32", seed=7)
    case.v_pool[:, 0] = 3.0
    case.v_pool[:, 1] = -5.0
    out = _decode(case).cpu()
    assert torch.allclose(out[:, :4], torch.tensor(3.0), atol=1e-6)
    assert torch.allclose(out[:, 4:], torch.tensor(-5.0), atol=1e-6)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("d,bs", [(64, 16), (128, 8), (128, 32)])
def test_append_bit_exact_over_whole_pool(dtype, d, bs):
    rng = np.random.default_rng(8)
    nb, hkv, n = 12, 4, 9
    pool_k = torch.full((nb, hkv, bs, d), 0, dtype=DT[dtype])
    pool_k.view(torch.uint8).fill_(0x5A)  # sentinel bytes: any stray write shows
    pool_v = pool_k.clone()
    kn, vn = randn((n, hkv, d), dtype, rng), randn((n, hkv, d), dtype, rng)
    slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int32)
    slots[[2, 5]] = -1  # padding tokens write nothing
    ek, ev = pa.kv_append(raw(pool_k), raw(pool_v), raw(kn), raw(vn), slots)
    gk, gv = pool_k.cuda(), pool_v.cuda()
    pkv.pkv_kv_append(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda(), gk, gv)
    assert np.array_equal(raw(gk).view(np.uint8), ek.view(np.uint8))
    assert np.array_equal(raw(gv).view(np.uint8), ev.view(np.uint8))


def test_copy_blocks_bit_exact():
    rng = np.random.default_rng(9)
    kp, vp = randn((10, 8, 16, 128), "bf16", rng), randn((10, 8, 16, 128), "bf16", rng)
    pairs = np.array([[1, 7], [3, 2], [9, 0]], dtype=np.int32)
    ek, ev = pa.copy_blocks(raw(kp), raw(vp), pairs)
    gk, gv = kp.cuda(), vp.cuda()
    pkv.pkv_copy_blocks(gk, gv, torch.from_numpy(pairs).cuda())
    assert np.array_equal(raw(gk), ek) and np.array_equal(raw(gv), ev)


def test_bad_block_id_is_reported_not_read():
    case = Case([40, 40], 8, 2, 128, 16, "bf16", seed=10)
    case.tables[1, 1] = case.nb + 1000  # outside the pool
    _decode(case)
    assert pkv.pkv_device_status(clear=True) == pkv._native.PKV_ERR_BAD_BLOCK
    assert pkv.pkv_device_status(clear=True) == 0
    kp = torch.zeros((4, 1, 16, 64), dtype=torch.float16, device="cuda")
    kn = torch.ones((1, 1, 64), dtype=torch.float16, device="cuda")
    pkv.pkv_kv_append(kn, kn, torch.tensor([4 * 16 + 3], dtype=torch.int32, device="cuda"), kp, kp.clone())
    assert pkv.pkv_device_status(clear=True) == pkv._native.PKV_ERR_BAD_BLOCK
    assert torch.count_nonzero(kp) == 0


def test_tiny_decode_step_end_to_end():
    """The smallest workload: 4 sequences of {1, 7, 16, 33} tokens, 4 heads,
    head_dim 64, fp32, 16-block pool; one append + attend step through the
    library's allocator, checked against the oracle's allocator model, append
    and attention (the 16 -> 17 sequence crosses a block boundary)."""
    from paged_kv_cache_406_b200 import workloads as W
    from paged_kv_cache_406_b200.cache import PagedKVCache
    w = W.WORKLOADS["tiny"]
    lens = W.seq_lens(w)
    nb = W.pool_blocks(w, lens)
    assert nb == 16
    order = W.free_order(nb, w.seed)
    shape = (nb, w.num_kv_heads, w.block_size, w.head_dim)
    k0 = W.normal(shape, torch.float32, W.pool_seed(w, 0))
    v0 = W.normal(shape, torch.float32, W.pool_seed(w, 1))
    maxb = 8
    cache = PagedKVCache(nb, w.num_kv_heads, w.head_dim, w.block_size, torch.float32, maxb, free_order=order,
                         k_pool=k0.cuda(), v_pool=v0.cuda())
    model = BlockAllocatorModel(nb, w.block_size, order)
    for b, L in enumerate(lens):
        cache.add(b, int(L))
        model.add(b, int(L))
    q = W.normal((4, 4, 64), torch.float32, W.step_seed(w, 0, 0))
    kn = W.normal((4, 4, 64), torch.float32, W.step_seed(w, 0, 1))
    vn = W.normal((4, 4, 64), torch.float32, W.step_seed(w, 0, 2))

    # attend-only on the pre-append state (sequence 0 has one token: out = v)
    tables = np.full((4, maxb), -1, dtype=np.int32)
    for b in range(4):
        t = model.block_table(b)
        tables[b, :len(t)] = t
    pre = pkv.pkv_paged_attention_decode(q.cuda(), cache.k_pool, cache.v_pool, torch.from_numpy(tables).cuda(),
                                         torch.from_numpy(lens.astype(np.int32)).cuda(), w.scale)
    ref_pre = pa.paged_decode_attention(raw(q), raw(k0), raw(v0), tables, lens, w.scale, "f32")
    assert_close(pre, ref_pre, "f32", "tiny pre-append")

    out = cache.decode_step(list(range(4)), q, kn, vn, w.scale)
    torch.cuda.synchronize()
    slots, cows = model.append_slots(list(range(4)))
    assert cows == []
    gslots = cache._meta_dev[:4].cpu().numpy()
    assert gslots.tolist() == slots
    ek, ev = pa.kv_append(raw(k0), raw(v0), raw(kn), raw(vn), np.array(slots))
    assert np.array_equal(raw(cache.k_pool), ek) and np.array_equal(raw(cache.v_pool), ev)
    for b in range(4):
        t = model.block_table(b)
        tables[b, :len(t)] = t
    post = lens + 1
    assert post.tolist() == [2, 8, 17, 34]
    ref = pa.paged_decode_attention(raw(q), ek, ev, tables, post, w.scale, "f32")
    assert_close(out, ref, "f32", "tiny step")
    assert TOL["f32"] == 1e-5
