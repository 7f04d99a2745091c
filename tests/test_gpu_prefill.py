"""GPU parity: causal paged prefill attention through the C-ABI against the
fp64 oracle (B200, tcgen05 kernel).

Tolerance: |gpu - oracle| <= 2e-3 * max(1, |oracle|) elementwise for bf16 /
fp16 K/V (fp32 output).  Every pool slot that no sequence owns (the tail of a
partial block, spare blocks) holds NaN, so a kernel that lets an unowned row
into the result cannot pass.
"""
import zlib

import numpy as np
import pytest
import torch

from helpers import DT, assert_close, raw
from oracle import paged_attention as pa
from oracle.block_allocator import BlockAllocatorModel

pytestmark = pytest.mark.gpu

import paged_kv_cache_406_b200 as pkv  # noqa: E402

D = 128


@pytest.fixture(autouse=True)
def _clean_status(native):
    pkv.pkv_device_status(clear=True)
    yield
    assert pkv.pkv_device_status(clear=True) == 0, "a kernel recorded a device error"


class PrefillCase:
    """Sequences of ``lens`` tokens whose last ``q_lens`` are the new chunk."""

    def __init__(self, lens, q_lens, hq, hkv, bs, dtype, seed, guard=3, k_ramp=0.0):
        rng = np.random.default_rng(seed)
        self.lens, self.q_lens = list(lens), list(q_lens)
        self.hq, self.hkv, self.bs, self.dtype = hq, hkv, bs, dtype
        need = sum(-(-L // bs) for L in self.lens)
        self.nb = need + guard
        model = BlockAllocatorModel(self.nb, bs, rng.permutation(self.nb))
        for b, L in enumerate(self.lens):
            model.add(b, L)
        self.maxb = max(1, max(len(model.block_table(b)) for b in range(len(self.lens))))
        self.tables = np.full((len(self.lens), self.maxb), -1, dtype=np.int32)
        shape = (self.nb, hkv, bs, D)
        k = torch.full(shape, float("nan"), dtype=torch.float32)
        v = torch.full(shape, float("nan"), dtype=torch.float32)
        for b, L in enumerate(self.lens):
            t = model.block_table(b)
            self.tables[b, :len(t)] = t
            kr = torch.from_numpy(rng.standard_normal((L, hkv, D), dtype=np.float32))
            vr = torch.from_numpy(rng.standard_normal((L, hkv, D), dtype=np.float32))
            if k_ramp:
                # scores that keep growing along the sequence: the running max
                # moves by more than the lazy-rescale threshold chunk after chunk
                kr = kr * 0.25 + k_ramp * torch.linspace(0, 1, L)[:, None, None]
            for i in range(L):
                k[t[i // bs], :, i % bs] = kr[i]
                v[t[i // bs], :, i % bs] = vr[i]
        self.k_pool, self.v_pool = k.to(DT[dtype]), v.to(DT[dtype])
        T = sum(self.q_lens)
        q = rng.standard_normal((T, hq, D), dtype=np.float32)
        if k_ramp:
            q = np.abs(q) * 0.5 + 1.0
        self.q = torch.from_numpy(q).to(DT[dtype])
        self.q_start = np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int32)
        self.scale = 1.0 / np.sqrt(D)

    def oracle(self):
        return pa.paged_prefill_attention(raw(self.q), raw(self.k_pool), raw(self.v_pool), self.tables,
                                          np.array(self.lens), np.array(self.q_lens), self.scale, self.dtype)

    def run(self, max_q_len=None, out=None, stage_v=True, workspace=None):
        dev = "cuda"
        res = pkv.pkv_paged_attention_prefill(
            self.q.to(dev), self.k_pool.to(dev), self.v_pool.to(dev), torch.from_numpy(self.tables).to(dev),
            torch.tensor(self.lens, dtype=torch.int32, device=dev), torch.from_numpy(self.q_start).to(dev),
            max(self.q_lens) if max_q_len is None else max_q_len, self.scale, out=out, stage_v=stage_v,
            workspace=workspace)
        torch.cuda.synchronize()
        return res


def _seed(*k):
    return zlib.crc32("-".join(map(str, k)).encode()) % 100000


@pytest.mark.parametrize("dtype,stage_v", [("bf16", True), ("bf16", False), ("f16", True)])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_prefill_matches_oracle(dtype, stage_v, g, bs):
    """Whole prompts, chunks behind earlier context, ragged tiles and chunks,
    lengths around the 128-key chunk edges; bf16 pools both with V staged as
    f16 (one f16 P·V pass) and without (P hi + lo over bf16 V)."""
    lens = [1, 130, 300, 129, 517, 64]
    q_lens = [1, 130, 77, 1, 45, 64]
    case = PrefillCase(lens, q_lens, 2 * g, 2, bs, dtype, _seed(dtype, g, bs))
    out = case.run(stage_v=stage_v)
    assert_close(out, case.oracle(), dtype, f"prefill {dtype} G{g} bs{bs} stage_v={stage_v}")


def test_bf16_v_beyond_f16_range_keeps_the_bf16_path():
    """A V value above 65504 has no f16 counterpart: the staged call must fall
    back to the two bf16 passes over the pool (bit for bit the unstaged
    result), and the next call on the same workspace, with values in range,
    must take the f16 pass again (its result then differs in the last bits
    from the unstaged one) - both within tolerance of the oracle."""
    lens, q_lens = [700, 300], [200, 300]
    big = PrefillCase(lens, q_lens, 8, 2, 16, "bf16", _seed("range"))
    t = big.tables[0, 1]
    big.v_pool[t, 0, 3, 5] = 131072.0  # token 19 of sequence 0, KV head 0, dim 5
    ws = torch.empty(pkv.pkv_prefill_workspace_size(2, 2, D, big.maxb, 16, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    staged = big.run(workspace=ws)
    plain = big.run(stage_v=False)
    assert torch.equal(staged, plain), "an out-of-range V must keep the bf16 hi + lo path"
    assert_close(staged, big.oracle(), "bf16", "V beyond the f16 range")
    small = PrefillCase(lens, q_lens, 8, 2, 16, "bf16", _seed("range"))
    staged = small.run(workspace=ws)
    plain = small.run(stage_v=False)
    assert not torch.equal(staged, plain), "values in range take the one-pass f16 P"
    ref = small.oracle()
    assert_close(staged, ref, "bf16", "staged after the fallback")
    assert_close(plain, ref, "bf16", "unstaged")


@pytest.mark.parametrize("dtype,stage_v", [("bf16", True), ("bf16", False), ("f16", True)])
@pytest.mark.parametrize("g", [1, 4])
def test_long_context_and_many_tiles(g, dtype, stage_v):
    """bf16 pools take P as hi + lo halves, or one f16 P over V staged as
    f16; f16 pools a single f16 P."""
    lens, q_lens = [1500, 700], [300, 700]
    case = PrefillCase(lens, q_lens, 2 * g, 2, 16, dtype, _seed("long", g, dtype))
    assert_close(case.run(stage_v=stage_v), case.oracle(), dtype, f"long {dtype} G{g} stage_v={stage_v}")


@pytest.mark.parametrize("dtype,stage_v", [("bf16", True), ("bf16", False), ("f16", True)])
def test_growing_scores_rescale_the_accumulator(dtype, stage_v):
    """Scores rise along the sequence so the running max moves by more than
    the lazy threshold in many chunks: every such move rescales O."""
    case = PrefillCase([900, 400], [200, 400], 8, 2, 16, dtype, _seed("ramp", dtype), k_ramp=12.0)
    ref = case.oracle()
    assert_close(case.run(stage_v=stage_v), ref, dtype, f"rescaled {dtype} stage_v={stage_v}")


def test_one_row_chunks_agree_with_decode():
    lens = [1, 15, 16, 17, 200, 1000]
    case = PrefillCase(lens, [1] * len(lens), 8, 2, 16, "bf16", _seed("decode"))
    pre = case.run()
    dec = pkv.pkv_paged_attention_decode(case.q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(),
                                         torch.from_numpy(case.tables).cuda(),
                                         torch.tensor(lens, dtype=torch.int32, device="cuda"), case.scale)
    torch.cuda.synchronize()
    ref = case.oracle()
    assert_close(pre, ref, "bf16", "prefill n=1")
    assert_close(dec, ref, "bf16", "decode")


def test_chunked_prefill_equals_one_shot():
    """A 600-token prompt fed as chunks of 128, 1, 300 and 171 tokens (each
    call seeing the pool as written so far) reproduces the one-shot rows."""
    L = 600
    whole = PrefillCase([L], [L], 8, 2, 16, "bf16", _seed("chunks"))
    ref = whole.oracle()
    full = whole.run()
    dev = "cuda"
    kp, vp, q = whole.k_pool.to(dev), whole.v_pool.to(dev), whole.q.to(dev)
    tables = torch.from_numpy(whole.tables).to(dev)
    pieces, start = [], 0
    for n in (128, 1, 300, 171):
        end = start + n
        out = pkv.pkv_paged_attention_prefill(q[start:end].contiguous(), kp, vp, tables,
                                              torch.tensor([end], dtype=torch.int32, device=dev),
                                              torch.tensor([0, n], dtype=torch.int32, device=dev), n, whole.scale)
        pieces.append(out)
        start = end
    torch.cuda.synchronize()
    chunked = torch.cat(pieces)
    assert_close(full, ref, "bf16", "one shot")
    assert_close(chunked, ref, "bf16", "chunked")


def test_empty_chunks_uncovered_rows_and_slack_tiles():
    """n = 0 sequences, rows no chunk owns (left untouched) and a max_q_len
    far above every chunk (the extra tiles exit)."""
    case = PrefillCase([40, 7, 90], [3, 0, 20], 8, 2, 8, "f16", _seed("empty"))
    dev = "cuda"
    T = sum(case.q_lens)
    q = torch.cat([case.q, torch.zeros((5, 8, D), dtype=case.q.dtype)]).to(dev)  # 5 rows owned by nobody
    out = torch.full((T + 5, 8, D), 7.0, dtype=torch.float32, device=dev)
    pkv.pkv_paged_attention_prefill(q, case.k_pool.to(dev), case.v_pool.to(dev),
                                    torch.from_numpy(case.tables).to(dev),
                                    torch.tensor(case.lens, dtype=torch.int32, device=dev),
                                    torch.from_numpy(case.q_start).to(dev), 1000, case.scale, out=out)
    torch.cuda.synchronize()
    assert_close(out[:T], case.oracle(), "f16", "owned rows")
    assert bool((out[T:] == 7.0).all()), "rows outside every chunk were written"


def test_chunk_longer_than_sequence_is_recorded():
    case = PrefillCase([10, 20], [5, 5], 4, 1, 16, "bf16", _seed("bad"))
    dev = "cuda"
    out = torch.full((10, 4, D), 3.0, device=dev)
    pkv.pkv_paged_attention_prefill(case.q.to(dev), case.k_pool.to(dev), case.v_pool.to(dev),
                                    torch.from_numpy(case.tables).to(dev),
                                    torch.tensor([3, 20], dtype=torch.int32, device=dev),  # 5 rows > 3 tokens
                                    torch.from_numpy(case.q_start).to(dev), 5, case.scale, out=out)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(clear=True) == pkv._native.PKV_ERR_INVALID_ARG
    assert bool((out[:5] == 3.0).all())
    ref = PrefillCase([10, 20], [5, 5], 4, 1, 16, "bf16", _seed("bad")).oracle()
    assert_close(out[5:], ref[5:], "bf16", "the valid sequence")


def test_unsupported_arguments_are_refused():
    dev = "cuda"
    kp = torch.zeros((4, 1, 16, D), dtype=torch.bfloat16, device=dev)
    tables = torch.zeros((1, 1), dtype=torch.int32, device=dev)
    lens = torch.ones(1, dtype=torch.int32, device=dev)
    qs = torch.tensor([0, 1], dtype=torch.int32, device=dev)
    with pytest.raises(pkv.PagedKVError) as e:  # fp32 pools: tensor cores take 16-bit operands only
        pkv.pkv_paged_attention_prefill(torch.zeros((1, 1, D), device=dev), kp.float(), kp.float(), tables, lens,
                                        qs, 1, 1.0)
    assert e.value.code == -4
    k64 = torch.zeros((4, 1, 16, 64), dtype=torch.bfloat16, device=dev)
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.pkv_paged_attention_prefill(torch.zeros((1, 1, 64), dtype=torch.bfloat16, device=dev), k64, k64,
                                        tables, lens, qs, 1, 1.0)
    assert e.value.code == -4
    for bad in (0.0, -0.5, float("nan")):  # the softmax takes the max of unscaled scores: scale > 0
        with pytest.raises(pkv.PagedKVError) as e:
            pkv.pkv_paged_attention_prefill(torch.zeros((1, 1, D), dtype=torch.bfloat16, device=dev), kp, kp,
                                            tables, lens, qs, 1, bad)
        assert e.value.code == -1
    with pytest.raises(pkv.PagedKVError) as e:  # group size 3
        pkv.pkv_paged_attention_prefill(torch.zeros((1, 3, D), dtype=torch.bfloat16, device=dev), kp, kp, tables,
                                        lens, qs, 1, 1.0)
    assert e.value.code == -4


@pytest.mark.parametrize("stage_v", [True, False])
def test_full_size_chunked_prefill_sampled_rows(stage_v):
    """The measured chunked-prefill batch (16 sequences, 512-row chunks behind
    U[0, 3584] cached tokens, 32 / 8 heads, bf16, block size 16), launched as
    the bench launches it (V staged as f16), and without staging; in every
    sequence, eight rows at and around the 128-row tile edges, every head,
    against the oracle, each as the one-row chunk at its position."""
    from paged_kv_cache_406_b200 import workloads as W
    w = W.WORKLOADS["prefill_llama3_8b"]
    dev = "cuda"
    B, hq, hkv, d, bs, n = w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.chunk_tokens
    ctx = W.seq_lens(w)
    L = ctx + n
    nb = W.pool_blocks(w, L)
    kp = W.pool_values((nb, hkv, bs, d), w, 0, device=dev)
    vp = W.pool_values((nb, hkv, bs, d), w, 1, device=dev)
    alloc = pkv.Allocator(nb, bs, W.free_order(nb, w.seed))
    for b in range(B):
        alloc.add(b, int(L[b]))
    maxb = -(-int(L.max()) // bs)
    tables, lens = alloc.block_tables(list(range(B)), maxb)
    q = W.normal((B * n, hq, d), w.torch_dtype, W.step_seed(w, 0, 0), device=dev)
    out = pkv.pkv_paged_attention_prefill(q, kp, vp, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev),
                                          torch.arange(0, B * n + 1, n, dtype=torch.int32, device=dev), n, w.scale,
                                          stage_v=stage_v)
    torch.cuda.synchronize()
    kc, vc, qc = raw(kp), raw(vp), raw(q)
    out = out.cpu()
    G = hq // hkv
    for b in range(B):
        kb, vb = kc[tables[b, :-(-int(L[b]) // bs)]], vc[tables[b, :-(-int(L[b]) // bs)]]
        for i in (0, 1, 31, 32, 127, 128, 300, n - 1):
            pos = int(ctx[b]) + i
            nblk = pos // bs + 1
            for g in range(hkv):
                ref = pa.paged_prefill_attention(qc[b * n + i:b * n + i + 1, g * G:(g + 1) * G],
                                                 kb[:nblk, g:g + 1], vb[:nblk, g:g + 1],
                                                 np.arange(nblk)[None], np.array([pos + 1]), np.array([1]),
                                                 w.scale, "bf16")
                got = out[b * n + i, g * G:(g + 1) * G].unsqueeze(0)
                assert_close(got, ref, "bf16", f"row {b}/{i} heads {g * G}..{g * G + G - 1}")


def test_repeated_concurrent_and_captured_calls():
    """The persistent kernel draws tiles from counters inside the library
    that each launch's last CTA re-arms: 70 calls in a row (more than the
    64 counters), two calls overlapping on two streams, and a captured graph
    replayed five times all give the single call's result bit for bit."""
    a = PrefillCase([300, 129, 517], [300, 1, 45], 8, 2, 16, "bf16", _seed("repeat", "a"))
    b = PrefillCase([700, 64], [128, 64], 8, 2, 16, "f16", _seed("repeat", "b"))

    def args(c):
        dev = "cuda"
        return (c.q.to(dev), c.k_pool.to(dev), c.v_pool.to(dev), torch.from_numpy(c.tables).to(dev),
                torch.tensor(c.lens, dtype=torch.int32, device=dev), torch.from_numpy(c.q_start).to(dev),
                max(c.q_lens), c.scale)

    xa, xb = args(a), args(b)
    ref_a = pkv.pkv_paged_attention_prefill(*xa).clone()
    ref_b = pkv.pkv_paged_attention_prefill(*xb).clone()
    torch.cuda.synchronize()
    assert_close(ref_a, a.oracle(), "bf16", "single call a")
    assert_close(ref_b, b.oracle(), "f16", "single call b")

    out = torch.empty_like(ref_a)
    for _ in range(70):
        pkv.pkv_paged_attention_prefill(*xa, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_a), "70 calls in a row"

    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    oa, ob = torch.empty_like(ref_a), torch.empty_like(ref_b)
    torch.cuda.synchronize()
    for _ in range(5):
        with torch.cuda.stream(s1):
            pkv.pkv_paged_attention_prefill(*xa, out=oa)
        with torch.cuda.stream(s2):
            pkv.pkv_paged_attention_prefill(*xb, out=ob)
    torch.cuda.synchronize()
    assert torch.equal(oa, ref_a) and torch.equal(ob, ref_b), "calls on two streams"

    og = torch.zeros_like(ref_a)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        pkv.pkv_paged_attention_prefill(*xa, out=og)  # first call outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            pkv.pkv_paged_attention_prefill(*xa, out=og)
    for _ in range(5):
        og.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(og, ref_a), "graph replay"
