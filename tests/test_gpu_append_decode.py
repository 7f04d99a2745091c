"""GPU parity for the append and decode of one step in one call
(pkv_append_and_decode and its e4m3 form), the decode step of the vLLM paging
page §3 (phase 1: the new token into its slot; phase 2: attention over every
cached token, the new one included).

Each case checks three things on the same seeded inputs:
- the pools equal the oracle's append byte for byte;
- the outputs are within tolerance of the oracle's attention over the
  appended pools;
- pools and outputs are bit-identical to the two-call form (pkv_kv_append,
  then pkv_paged_attention_decode).
"""
import zlib

import numpy as np
import pytest
import torch

from helpers import DT, Case, assert_close, randn, raw
from oracle import fp8 as of
from oracle import paged_attention as pa

pytestmark = pytest.mark.gpu

import paged_kv_cache_406_b200 as pkv  # noqa: E402


@pytest.fixture(autouse=True)
def _clean_status(native):
    pkv.pkv_device_status(clear=True)
    yield
    assert pkv.pkv_device_status(clear=True) == 0, "a kernel recorded a device error"


def _lens(bs):
    return [0, 1, bs - 1, bs, bs + 1, 2 * bs + 3, 100, 255, 256, 511, 512, 1023, 1024]


def _grow(case: Case, skip=()):
    """Slots of one new token per sequence (the oracle's allocator model),
    the tables and lengths after it; sequences in ``skip`` get slot -1 (a
    padding token) and keep their length."""
    ids = [b for b in range(case.B) if b not in skip]
    got, cows = case.model.append_slots(ids)
    assert cows == []
    slots = np.full(case.B, -1, dtype=np.int32)
    slots[ids] = got
    maxb = max(len(case.model.block_table(b)) for b in range(case.B))
    tables = np.full((case.B, maxb), -1, dtype=np.int32)
    for b in range(case.B):
        t = case.model.block_table(b)
        tables[b, :len(t)] = t
    lens = np.array([case.model.seq_len(b) for b in range(case.B)], dtype=np.int64)
    return slots, tables, lens


@pytest.mark.parametrize("dtype,d,g,bs,pt", [
    ("bf16", 128, 4, 16, 0),     # tensor-core kernel, 512-token partitions
    ("bf16", 128, 4, 16, 64),    # many partitions: the merge kernel on most sequences
    ("f16", 128, 8, 32, 0),
    ("bf16", 64, 2, 8, 0),
    ("f32", 128, 4, 16, 0),      # CUDA-core kernel
    ("f16", 128, 1, 16, 128),    # CUDA-core kernel, G = 1
])
def test_append_and_decode_matches_oracle_and_two_calls(dtype, d, g, bs, pt):
    hkv = 2
    case = Case(_lens(bs), g * hkv, hkv, d, bs, dtype, seed=zlib.crc32(f"ad{dtype}{d}{g}{bs}{pt}".encode()) % 1000,
                guard=8)
    rng = np.random.default_rng(case.B + d + g)
    slots, tables, lens = _grow(case, skip=(3,))
    kn, vn = randn((case.B, hkv, d), dtype, rng), randn((case.B, hkv, d), dtype, rng)
    ek, ev = pa.kv_append(raw(case.k_pool), raw(case.v_pool), raw(kn), raw(vn), slots)
    ref = pa.paged_decode_attention(raw(case.q), ek, ev, tables, lens, case.scale, dtype)

    dev = dict(kn=kn.cuda(), vn=vn.cuda(), slots=torch.from_numpy(slots).cuda(), q=case.q.cuda(),
               tables=torch.from_numpy(tables).cuda(), lens=torch.from_numpy(lens.astype(np.int32)).cuda())
    fk, fv = case.k_pool.cuda(), case.v_pool.cuda()
    out = pkv.pkv_append_and_decode(dev["kn"], dev["vn"], dev["slots"], dev["q"], fk, fv, dev["tables"], dev["lens"],
                                    case.scale, partition_tokens=pt)
    tk, tv = case.k_pool.cuda(), case.v_pool.cuda()
    pkv.pkv_kv_append(dev["kn"], dev["vn"], dev["slots"], tk, tv)
    two = pkv.pkv_paged_attention_decode(dev["q"], tk, tv, dev["tables"], dev["lens"], case.scale,
                                         partition_tokens=pt)
    torch.cuda.synchronize()
    assert np.array_equal(raw(fk), ek) and np.array_equal(raw(fv), ev), "pool differs from the oracle's append"
    assert torch.equal(fk, tk) and torch.equal(fv, tv)
    assert torch.equal(out, two), "one-call and two-call results differ"
    assert_close(out, ref, dtype, f"append+decode {dtype} D{d} G{g} bs{bs} pt{pt}")


def test_no_new_rows_is_plain_decode():
    case = Case(_lens(16), 8, 2, 128, 16, "bf16", seed=31)
    d = case.device()
    empty = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    none = torch.empty((0,), dtype=torch.int32, device="cuda")
    k0 = d["k_pool"].clone()
    out = pkv.pkv_append_and_decode(empty, empty, none, d["q"], d["k_pool"], d["v_pool"], d["block_tables"],
                                    d["seq_lens"], case.scale)
    ref = pkv.pkv_paged_attention_decode(d["q"], d["k_pool"], d["v_pool"], d["block_tables"], d["seq_lens"],
                                         case.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, ref) and torch.equal(d["k_pool"], k0)


def test_empty_batch_still_appends():
    rng = np.random.default_rng(32)
    kp = torch.zeros((6, 2, 16, 128), dtype=torch.float16)
    kn, vn = randn((3, 2, 128), "f16", rng), randn((3, 2, 128), "f16", rng)
    slots = np.array([5, 17, 90], dtype=np.int32)
    ek, ev = pa.kv_append(raw(kp), raw(kp), raw(kn), raw(vn), slots)
    gk, gv = kp.cuda(), kp.cuda()
    q = torch.empty((0, 8, 128), dtype=torch.float16, device="cuda")
    tables = torch.empty((0, 4), dtype=torch.int32, device="cuda")
    lens = torch.empty((0,), dtype=torch.int32, device="cuda")
    out = pkv.pkv_append_and_decode(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda(), q, gk, gv, tables, lens,
                                    0.1)
    torch.cuda.synchronize()
    assert out.shape == (0, 8, 128)
    assert np.array_equal(raw(gk), ek) and np.array_equal(raw(gv), ev)


def test_rejected_call_writes_nothing():
    """Arguments are checked before any launch: a bad scale fails the call
    and the new rows are not written."""
    case = Case([40, 7], 8, 2, 128, 16, "bf16", seed=33, guard=4)
    rng = np.random.default_rng(33)
    slots, tables, lens = _grow(case)
    kn, vn = randn((2, 2, 128), "bf16", rng), randn((2, 2, 128), "bf16", rng)
    fk, fv = case.k_pool.cuda(), case.v_pool.cuda()
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_append_and_decode(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda(), case.q.cuda(), fk, fv,
                                  torch.from_numpy(tables).cuda(), torch.from_numpy(lens.astype(np.int32)).cuda(),
                                  float("inf"))
    torch.cuda.synchronize()
    assert torch.equal(fk.cpu(), case.k_pool) and torch.equal(fv.cpu(), case.v_pool)


@pytest.mark.parametrize("g,bs", [(4, 16), (8, 8)])
def test_append_and_decode_fp8_matches_oracle_and_two_calls(g, bs):
    hkv, d = 2, 128
    rng = np.random.default_rng(40 + g + bs)
    case = Case(_lens(bs), g * hkv, hkv, d, bs, "f16", seed=41 + g, guard=8)
    k_scale, v_scale = 0.5, 0.25
    kc = torch.from_numpy(rng.integers(0, 0x7F, size=case.k_pool.shape, dtype=np.uint8))  # finite codes
    vc = torch.from_numpy(rng.integers(0, 0x7F, size=case.v_pool.shape, dtype=np.uint8))
    slots, tables, lens = _grow(case, skip=(5,))
    kn, vn = randn((case.B, hkv, d), "f16", rng), randn((case.B, hkv, d), "f16", rng)
    ek, ev = of.kv_append_fp8(kc.numpy(), vc.numpy(), raw(kn), raw(vn), slots, k_scale, v_scale)
    ref = of.paged_decode_attention_fp8(raw(case.q), ek, ev, tables, lens, case.scale, k_scale, v_scale)

    dev = dict(kn=kn.cuda(), vn=vn.cuda(), slots=torch.from_numpy(slots).cuda(), q=case.q.cuda(),
               tables=torch.from_numpy(tables).cuda(), lens=torch.from_numpy(lens.astype(np.int32)).cuda())
    fk, fv = kc.cuda(), vc.cuda()
    out = pkv.pkv_append_and_decode_fp8(dev["kn"], dev["vn"], dev["slots"], dev["q"], fk, fv, dev["tables"],
                                        dev["lens"], case.scale, k_scale, v_scale)
    tk, tv = kc.cuda(), vc.cuda()
    pkv.pkv_kv_append_fp8(dev["kn"], dev["vn"], dev["slots"], tk, tv, k_scale, v_scale)
    two = pkv.pkv_paged_attention_decode_fp8(dev["q"], tk, tv, dev["tables"], dev["lens"], case.scale, k_scale,
                                             v_scale)
    torch.cuda.synchronize()
    assert np.array_equal(fk.cpu().numpy(), ek) and np.array_equal(fv.cpu().numpy(), ev)
    assert torch.equal(fk, tk) and torch.equal(fv, tv)
    assert torch.equal(out, two)
    assert_close(out, ref, "f16", f"append+decode e4m3 G{g} bs{bs}")


def test_bound_call_equals_the_plain_call():
    """bind_append_and_decode: the call checked and marshalled once, issued
    twice, gives the plain call's pools and outputs bit for bit."""
    case = Case([5, 300, 1030, 2049], 8, 2, 128, 16, "bf16", seed=71)
    slots, tables, lens = _grow(case)
    rng = np.random.default_rng(72)
    kn, vn = randn((case.B, 2, 128), "bf16", rng), randn((case.B, 2, 128), "bf16", rng)
    dev = "cuda"
    args = dict(k_new=kn.to(dev), v_new=vn.to(dev), slot_mapping=torch.from_numpy(slots).to(dev), q=case.q.to(dev),
                block_tables=torch.from_numpy(tables).to(dev), seq_lens=torch.from_numpy(lens.astype(np.int32)).to(dev))
    kp1, vp1 = case.k_pool.to(dev), case.v_pool.to(dev)
    kp2, vp2 = kp1.clone(), vp1.clone()
    want = pkv.pkv_append_and_decode(args["k_new"], args["v_new"], args["slot_mapping"], args["q"], kp1, vp1,
                                     args["block_tables"], args["seq_lens"], case.scale)
    ws = torch.empty(pkv.pkv_decode_workspace_size(case.B, 8, 2, 128, tables.shape[1], 16, 0), dtype=torch.uint8,
                     device=dev)
    out = torch.full_like(want, float("nan"))
    call = pkv.bind_append_and_decode(args["k_new"], args["v_new"], args["slot_mapping"], args["q"], kp2, vp2,
                                      args["block_tables"], args["seq_lens"], case.scale, out, ws)
    for _ in range(2):
        got = call()
        torch.cuda.synchronize()
        assert got is out
        assert torch.equal(out, want)
    assert torch.equal(kp1, kp2) and torch.equal(vp1, vp2)
