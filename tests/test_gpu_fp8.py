"""GPU parity of the FP8 (e4m3) KV cache against the oracle (B200): the
quantising append byte for byte over the whole pool, decode attention over
e4m3 pools within the 16-bit tolerance, and agreement with the 16-bit kernel
on the same dequantised values."""
import zlib

import numpy as np
import pytest
import torch

from helpers import TOL, assert_close, raw
from oracle import fp8
from oracle.block_allocator import BlockAllocatorModel

pytestmark = pytest.mark.gpu

import paged_kv_cache_406_b200 as pkv  # noqa: E402


@pytest.fixture(autouse=True)
def _clean_status(native):
    pkv.pkv_device_status(clear=True)
    yield
    assert pkv.pkv_device_status(clear=True) == 0, "a kernel recorded a device error"


def _finite_codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 0x01  # no NaN codes
    return c


class Fp8Case:
    def __init__(self, lens, hq, hkv, bs, seed, k_scale=0.25, v_scale=0.5, d=128):
        rng = np.random.default_rng(seed)
        self.lens = np.asarray(lens, dtype=np.int64)
        self.hq, self.hkv, self.bs, self.d = hq, hkv, bs, d
        need = int(sum(-(-int(L) // bs) for L in lens))
        self.nb = need + 3
        model = BlockAllocatorModel(self.nb, bs, rng.permutation(self.nb))
        for b, L in enumerate(lens):
            model.add(b, int(L))
        self.maxb = max(1, max(len(model.block_table(b)) for b in range(len(lens))))
        self.tables = np.full((len(lens), self.maxb), -1, dtype=np.int32)
        for b in range(len(lens)):
            t = model.block_table(b)
            self.tables[b, :len(t)] = t
        self.kc = _finite_codes(rng, (self.nb, hkv, bs, d))
        self.vc = _finite_codes(rng, (self.nb, hkv, bs, d))
        self.q = torch.from_numpy(rng.standard_normal((len(lens), hq, d), dtype=np.float32)).to(torch.float16)
        self.k_scale, self.v_scale = k_scale, v_scale
        self.scale = 1.0 / np.sqrt(d)

    def oracle(self):
        return fp8.paged_decode_attention_fp8(raw(self.q), self.kc, self.vc, self.tables, self.lens, self.scale,
                                              self.k_scale, self.v_scale)

    def gpu(self, pt=0):
        out = pkv.pkv_paged_attention_decode_fp8(
            self.q.cuda(), torch.from_numpy(self.kc).cuda(), torch.from_numpy(self.vc).cuda(),
            torch.from_numpy(self.tables).cuda(), torch.from_numpy(self.lens.astype(np.int32)).cuda(), self.scale,
            self.k_scale, self.v_scale, partition_tokens=pt)
        torch.cuda.synchronize()
        return out


@pytest.mark.parametrize("src", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fp8_append_bit_exact_over_whole_pool(src, bs):
    rng = np.random.default_rng(zlib.crc32(f"{src}{bs}".encode()))
    nb, hkv, d, n = 10, 4, 128, 11
    kp = np.full((nb, hkv, bs, d), 0x5A, dtype=np.uint8)  # sentinel codes
    vp = kp.copy()
    dt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[src]
    kn = torch.from_numpy(rng.standard_normal((n, hkv, d), dtype=np.float32) * 60).to(dt)
    vn = torch.from_numpy(rng.standard_normal((n, hkv, d), dtype=np.float32) * 3).to(dt)
    kn[0, 0, :4] = torch.tensor([500.0, -1000.0, 1e-9, 0.0], dtype=dt)  # saturation, underflow, zero
    slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int32)
    slots[3] = -1
    k_scale, v_scale = 0.375, 0.0625
    ek, ev = fp8.kv_append_fp8(kp, vp, kn.float().numpy(), vn.float().numpy(), slots, k_scale, v_scale)
    gk, gv = torch.from_numpy(kp).cuda(), torch.from_numpy(vp).cuda()
    pkv.pkv_kv_append_fp8(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda(), gk, gv, k_scale, v_scale)
    assert np.array_equal(gk.cpu().numpy(), ek)
    assert np.array_equal(gv.cpu().numpy(), ev)


@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fp8_decode_matches_oracle(g, bs):
    lens = [0, 1, bs - 1, bs + 1, 100, 511, 512, 513, 1025, 2000]
    case = Fp8Case(lens, 2 * g, 2, bs, seed=zlib.crc32(f"fp8{g}{bs}".encode()))
    assert_close(case.gpu(), case.oracle(), "f16", f"fp8 G{g} bs{bs}")


def test_fp8_single_token_and_split_sizes():
    case = Fp8Case([1, 700, 1300], 8, 2, 16, seed=5, k_scale=2.0, v_scale=0.125)
    ref = case.oracle()
    for pt in (16, 64, 512, 8192):
        assert_close(case.gpu(pt), ref, "f16", f"partition {pt}")
    out = case.gpu()
    blk = case.tables[0, 0]
    v = torch.from_numpy(fp8.e4m3_decode(case.vc[blk, 0, 0]) * case.v_scale).float()
    assert torch.equal(out[0, 0].cpu(), v), "one token: out = v_scale * e4m3(v) exactly"


def test_fp8_agrees_with_f16_kernel_on_dequantised_pools():
    case = Fp8Case([37, 600, 1500], 16, 4, 16, seed=6, k_scale=0.5, v_scale=0.25)  # powers of two: exact in f16
    kf = torch.from_numpy(fp8.e4m3_decode(case.kc) * case.k_scale).to(torch.float16).cuda()
    vf = torch.from_numpy(fp8.e4m3_decode(case.vc) * case.v_scale).to(torch.float16).cuda()
    ref16 = pkv.pkv_paged_attention_decode(case.q.cuda(), kf, vf, torch.from_numpy(case.tables).cuda(),
                                           torch.from_numpy(case.lens.astype(np.int32)).cuda(), case.scale)
    out8 = case.gpu()
    assert torch.max(torch.abs(out8 - ref16)).item() < TOL["f16"]


def test_fp8_rejects_unsupported_shapes():
    case = Fp8Case([5], 4, 1, 16, seed=7, d=64)
    with pytest.raises(pkv.PagedKVError):
        case.gpu()


def test_llama3_8b_fp8_decode_step_full_size(native):
    """One append + attend step of the Llama-3-8B-shaped batch with an e4m3 KV
    cache through PagedKVCache, with distinct K and V scales: slots equal the
    allocator model's; both pools equal the oracle's (pristine pool + the
    oracle's quantising append for every sequence) byte for byte; attention
    of every sequence and head is within tolerance."""
    from paged_kv_cache_406_b200 import workloads as W
    from paged_kv_cache_406_b200.cache import PagedKVCache
    w = W.WORKLOADS["llama3_8b_fp8"]
    k_scale, v_scale = w.kv_scale, 2 * w.kv_scale
    lens = W.seq_lens(w)
    nb = W.pool_blocks(w, lens)
    order = W.free_order(nb, w.seed)
    shape = (nb, w.num_kv_heads, w.block_size, w.head_dim)
    k0 = W.pool_values(shape, w, 0, device="cuda")
    v0 = W.pool_values(shape, w, 1, device="cuda")
    maxb = -(-(int(lens.max()) + 1) // w.block_size)
    cache = PagedKVCache(nb, w.num_kv_heads, w.head_dim, w.block_size, w.torch_dtype, maxb, free_order=order,
                         k_pool=k0.clone(), v_pool=v0.clone(), k_scale=k_scale, v_scale=v_scale)
    model = BlockAllocatorModel(nb, w.block_size, order)
    ids = list(range(w.num_seqs))
    for b in ids:
        cache.add(b, int(lens[b]))
        model.add(b, int(lens[b]))
    q = W.normal((w.num_seqs, w.num_q_heads, w.head_dim), w.io_dtype, W.step_seed(w, 0, 0))
    kn = W.normal((w.num_seqs, w.num_kv_heads, w.head_dim), w.io_dtype, W.step_seed(w, 0, 1))
    vn = W.normal((w.num_seqs, w.num_kv_heads, w.head_dim), w.io_dtype, W.step_seed(w, 0, 2))
    out = cache.decode_step(ids, q, kn, vn, w.scale).cpu()
    torch.cuda.synchronize()
    slots, _ = model.append_slots(ids)
    assert cache._meta_dev[:w.num_seqs].cpu().numpy().tolist() == slots
    kc, vc = fp8.kv_append_fp8(k0.view(torch.uint8).cpu().numpy(), v0.view(torch.uint8).cpu().numpy(),
                               kn.float().numpy(), vn.float().numpy(), np.array(slots), k_scale, v_scale)
    assert np.array_equal(cache.k_pool.view(torch.uint8).cpu().numpy(), kc), "K pool differs from the oracle's"
    assert np.array_equal(cache.v_pool.view(torch.uint8).cpu().numpy(), vc), "V pool differs from the oracle's"
    qr = raw(q)
    for b in ids:
        tab = np.asarray(model.block_table(b))
        local = np.arange(len(tab), dtype=np.int32)[None]
        ref = fp8.paged_decode_attention_fp8(qr[b:b + 1], kc[tab], vc[tab], local, np.array([model.seq_len(b)]),
                                             w.scale, k_scale, v_scale)
        assert_close(out[b:b + 1], ref, "f16", f"fp8 llama3 seq {b}")
    assert w.group == 4
