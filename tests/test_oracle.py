"""Pins for the fp64 attention / append / copy oracle (CPU only).

Each test ties the oracle to something other than itself: brute force written
with explicit loops, PyTorch's CPU scaled-dot-product attention in float64 as a
library special case, closed forms (L = 1, L = 2, constant V, scale 0, a
single dominant score), and invariants the definition forces (any permutation
of physical blocks, any block size, either pool layout, weights summing to one,
split-partition rescaling).  A dropped scale, a sign error, a wrong GQA head
index, an off-by-one in the gather or a transposed operand each fails at least
one of them; ``test_planted_mistakes_are_caught`` checks that directly.
"""
import math

import numpy as np
import pytest
import torch

from oracle import paged_attention as pa


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _scatter(contig, block_size, perm, layout="NHBD", num_blocks=None):
    """Lay contiguous per-sequence rows ``[L_b, H, D]`` into a pool.

    Sequence b's logical blocks take the next entries of ``perm``; returns
    (pool, tables).  Written independently of the oracle's gather."""
    H, D = contig[0].shape[1:]
    nblk = [-(-len(c) // block_size) for c in contig]
    total = num_blocks or max(sum(nblk), 1)
    dtype = contig[0].dtype
    if layout == "NHBD":
        pool = np.zeros((total, H, block_size, D), dtype=dtype)
    else:
        pool = np.zeros((total, block_size, H, D), dtype=dtype)
    tables = np.full((len(contig), max(max(nblk), 1)), -1, dtype=np.int32)
    k = 0
    for b, c in enumerate(contig):
        for j in range(nblk[b]):
            p = perm[k]
            k += 1
            tables[b, j] = p
            for o in range(block_size):
                t = j * block_size + o
                if t >= len(c):
                    break
                if layout == "NHBD":
                    pool[p, :, o, :] = c[t]
                else:
                    pool[p, o, :, :] = c[t]
    return pool, tables


def _brute(q, Ks, Vs, scale, G):
    """Contiguous attention with explicit Python loops and math.exp."""
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = len(Ks[b])
        for h in range(Hq):
            g = h // G
            s = []
            for t in range(L):
                acc = 0.0
                for d in range(D):
                    acc += float(q[b, h, d]) * float(Ks[b][t, g, d])
                s.append(acc * scale)
            if not s:
                continue
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            tot = sum(e)
            for d in range(D):
                out[b, h, d] = sum(e[t] * float(Vs[b][t, g, d]) for t in range(L)) / tot
    return out


def _random_case(rng, B, Hq, Hkv, D, lens, dtype=np.float64):
    q = rng.standard_normal((B, Hq, D)).astype(dtype)
    Ks = [rng.standard_normal((L, Hkv, D)).astype(dtype) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D)).astype(dtype) for L in lens]
    return q, Ks, Vs


def _run_paged(q, Ks, Vs, scale, bs, perm_seed, layout="NHBD", dtype="f32"):
    lens = [len(k) for k in Ks]
    nb = sum(-(-L // bs) for L in lens)
    perm = np.random.default_rng(perm_seed).permutation(max(nb, 1))
    kp, tables = _scatter(Ks, bs, perm, layout)
    vp, _ = _scatter(Vs, bs, perm, layout)
    return pa.paged_decode_attention(q, kp, vp, tables, np.array(lens), scale, dtype, layout)


def test_to_f64_bf16_bit_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x7F80, 0x4049], dtype=np.uint16)
    want = [1.0, -2.0, 1.0 + 2.0 ** -7, 0.0, -0.0, math.inf, 3.140625]
    got = pa.to_f64(bits, "bf16")
    assert got.tolist() == want
    # library cross-check: torch's own bf16 -> float64 widening
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, lib)


def test_to_f64_f16_and_f32():
    x = np.array([1.5, -0.25, 65504.0], dtype=np.float16)
    assert pa.to_f64(x, "f16").tolist() == [1.5, -0.25, 65504.0]
    y = np.array([np.float32(0.1)], dtype=np.float32)
    assert pa.to_f64(y, "f32")[0] == float(np.float32(0.1))


def test_matches_brute_force_loops():
    rng = np.random.default_rng(1)
    lens = [1, 5, 16, 17, 33]
    q, Ks, Vs = _random_case(rng, len(lens), 4, 2, 8, lens, np.float32)
    scale = 1 / math.sqrt(8)
    got = _run_paged(q, Ks, Vs, scale, bs=4, perm_seed=2)
    want = _brute(q, Ks, Vs, scale, G=2)
    assert np.max(np.abs(got - want)) < 1e-12


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (32, 8)])
def test_matches_torch_sdpa_fp64(Hq, Hkv):
    rng = np.random.default_rng(3)
    lens = [3, 40, 64, 97]
    D = 16
    q, Ks, Vs = _random_case(rng, len(lens), Hq, Hkv, D, lens, np.float32)
    scale = 0.37
    got = _run_paged(q, Ks, Vs, scale, bs=16, perm_seed=4)
    G = Hq // Hkv
    for b, L in enumerate(lens):
        qt = torch.from_numpy(q[b].astype(np.float64))[None, :, None, :]  # [1,Hq,1,D]
        k = torch.from_numpy(Ks[b].astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
        v = torch.from_numpy(Vs[b].astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, k, v, scale=scale)[0, :, 0, :].numpy()
        assert np.max(np.abs(got[b] - ref)) < 1e-12


def test_invariant_under_block_permutation():
    rng = np.random.default_rng(5)
    lens = [7, 31, 64, 100]
    q, Ks, Vs = _random_case(rng, len(lens), 8, 4, 16, lens, np.float32)
    a = _run_paged(q, Ks, Vs, 0.25, bs=8, perm_seed=10)
    b = _run_paged(q, Ks, Vs, 0.25, bs=8, perm_seed=11)
    assert np.array_equal(a, b)


def test_invariant_under_block_size():
    rng = np.random.default_rng(6)
    lens = [1, 9, 33, 70]
    q, Ks, Vs = _random_case(rng, len(lens), 4, 2, 16, lens, np.float32)
    outs = [_run_paged(q, Ks, Vs, 0.3, bs=bs, perm_seed=bs) for bs in (1, 8, 16, 32)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_invariant_under_layout():
    rng = np.random.default_rng(7)
    lens = [12, 50]
    q, Ks, Vs = _random_case(rng, len(lens), 4, 4, 8, lens, np.float32)
    a = _run_paged(q, Ks, Vs, 0.5, bs=16, perm_seed=1, layout="NHBD")
    b = _run_paged(q, Ks, Vs, 0.5, bs=16, perm_seed=1, layout="NBHD")
    assert np.array_equal(a, b)


def test_softmax_weights_sum_to_one():
    rng = np.random.default_rng(8)
    for L in (1, 2, 17, 1000):
        keys = rng.standard_normal((L, 32))
        w = pa.attention_weights(rng.standard_normal(32), keys, 1 / math.sqrt(32))
        assert np.all(w >= 0)
        assert abs(w.sum() - 1.0) < 1e-12


def test_single_token_returns_v_exactly():
    rng = np.random.default_rng(9)
    q, Ks, Vs = _random_case(rng, 3, 8, 2, 16, [1, 1, 1], np.float32)
    got = _run_paged(q, Ks, Vs, 0.125, bs=16, perm_seed=3)
    for b in range(3):
        for h in range(8):
            assert np.array_equal(got[b, h], Vs[b][0, h // 4].astype(np.float64))


def test_two_tokens_logistic_closed_form():
    rng = np.random.default_rng(10)
    q, Ks, Vs = _random_case(rng, 1, 2, 1, 4, [2], np.float32)
    scale = 0.7
    got = _run_paged(q, Ks, Vs, scale, bs=1, perm_seed=0)
    for h in range(2):
        s0 = scale * sum(float(q[0, h, d]) * float(Ks[0][0, 0, d]) for d in range(4))
        s1 = scale * sum(float(q[0, h, d]) * float(Ks[0][1, 0, d]) for d in range(4))
        w1 = 1.0 / (1.0 + math.exp(s0 - s1))
        want = (1 - w1) * Vs[0][0, 0].astype(np.float64) + w1 * Vs[0][1, 0].astype(np.float64)
        assert np.max(np.abs(got[0, h] - want)) < 1e-14


def test_constant_v_gives_constant():
    rng = np.random.default_rng(11)
    lens = [5, 300]
    q, Ks, _ = _random_case(rng, 2, 4, 2, 8, lens, np.float32)
    Vs = [np.full((L, 2, 8), 1.75, dtype=np.float32) for L in lens]
    got = _run_paged(q, Ks, Vs, 0.3, bs=16, perm_seed=5)
    assert np.max(np.abs(got - 1.75)) < 1e-14


def test_scale_zero_gives_mean_of_v():
    rng = np.random.default_rng(12)
    lens = [6, 45]
    q, Ks, Vs = _random_case(rng, 2, 2, 1, 8, lens, np.float32)
    got = _run_paged(q, Ks, Vs, 0.0, bs=8, perm_seed=6)
    for b in range(2):
        assert np.max(np.abs(got[b, 0] - Vs[b][:, 0].astype(np.float64).mean(axis=0))) < 1e-14


def test_dominant_score_selects_its_value():
    """A huge scale turns the softmax into an argmax: the output is the V row
    of the largest score (a sign error would pick the smallest)."""
    rng = np.random.default_rng(13)
    q, Ks, Vs = _random_case(rng, 1, 1, 1, 8, [20], np.float32)
    got = _run_paged(q, Ks, Vs, 1e4, bs=4, perm_seed=7)
    s = Ks[0][:, 0].astype(np.float64) @ q[0, 0].astype(np.float64)
    assert np.max(np.abs(got[0, 0] - Vs[0][int(np.argmax(s)), 0])) < 1e-12


def test_gqa_groups_are_contiguous():
    """Query heads 0..G-1 read KV head 0, the next G read KV head 1, ..."""
    lens = [9]
    rng = np.random.default_rng(14)
    q, Ks, _ = _random_case(rng, 1, 6, 3, 4, lens, np.float32)
    V = np.zeros((9, 3, 4), dtype=np.float32)
    for g in range(3):
        V[:, g, :] = 10.0 * (g + 1)
    got = _run_paged(q, Ks, [V], 0.5, bs=4, perm_seed=8)
    for h in range(6):
        assert np.allclose(got[0, h], 10.0 * (h // 2 + 1), atol=1e-12)


def test_zero_length_gives_zeros():
    q = np.ones((2, 2, 4), dtype=np.float32)
    pool = np.ones((2, 2, 4, 4), dtype=np.float32)
    tables = np.array([[0], [1]], dtype=np.int32)
    out = pa.paged_decode_attention(q, pool, pool, tables, np.array([0, 3]), 1.0, "f32")
    assert np.array_equal(out[0], np.zeros((2, 4)))
    assert np.allclose(out[1], 1.0)


def test_bf16_inputs_match_widened_float_inputs():
    rng = np.random.default_rng(15)
    lens = [10, 40]
    q, Ks, Vs = _random_case(rng, 2, 4, 1, 8, lens, np.float32)
    qb = _bf16_bits(q)
    Kb = [_bf16_bits(k) for k in Ks]
    Vb = [_bf16_bits(v) for v in Vs]
    got = _run_paged(qb, Kb, Vb, 0.3, bs=8, perm_seed=9, dtype="bf16")
    widen = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    want = _brute(widen(qb), [widen(k) for k in Kb], [widen(v) for v in Vb], 0.3, G=4)
    assert np.max(np.abs(got - want)) < 1e-12


def test_append_writes_exactly_the_slots():
    rng = np.random.default_rng(16)
    NB, H, bs, D = 5, 2, 4, 3
    kp = rng.standard_normal((NB, H, bs, D)).astype(np.float32)
    vp = rng.standard_normal((NB, H, bs, D)).astype(np.float32)
    kn = rng.standard_normal((4, H, D)).astype(np.float32)
    vn = rng.standard_normal((4, H, D)).astype(np.float32)
    slots = np.array([3, -1, 17, 8], dtype=np.int32)
    k2, v2 = pa.kv_append(kp, vp, kn, vn, slots)
    changed = set()
    for i, s in enumerate(slots):
        if s < 0:
            continue
        p, o = s // bs, s % bs
        changed.add((p, o))
        assert np.array_equal(k2[p, :, o, :], kn[i])
        assert np.array_equal(v2[p, :, o, :], vn[i])
    for p in range(NB):
        for o in range(bs):
            if (p, o) not in changed:
                assert np.array_equal(k2[p, :, o, :], kp[p, :, o, :])
                assert np.array_equal(v2[p, :, o, :], vp[p, :, o, :])
    # inputs untouched
    assert not np.shares_memory(k2, kp)


def test_append_then_gather_reads_new_token_last():
    rng = np.random.default_rng(17)
    bs = 4
    kp = rng.standard_normal((3, 1, bs, 2)).astype(np.float32)
    table = np.array([2, 0], dtype=np.int32)
    kn = rng.standard_normal((1, 1, 2)).astype(np.float32)
    # sequence of 5 tokens grows to 6: slot of position 5 is block table[1], offset 1
    k2, _ = pa.kv_append(kp, kp, kn, kn, np.array([table[1] * bs + 1]))
    rows = pa.gather_sequence(k2, table, 6)
    assert np.array_equal(rows[5], kn[0])
    assert np.array_equal(rows[:5], pa.gather_sequence(kp, table, 5))


def test_copy_blocks():
    rng = np.random.default_rng(18)
    kp = rng.standard_normal((4, 2, 2, 2)).astype(np.float32)
    vp = rng.standard_normal((4, 2, 2, 2)).astype(np.float32)
    k2, v2 = pa.copy_blocks(kp, vp, np.array([[1, 3], [0, 2]]))
    assert np.array_equal(k2[3], kp[1]) and np.array_equal(v2[3], vp[1])
    assert np.array_equal(k2[2], kp[0]) and np.array_equal(v2[2], vp[0])
    assert np.array_equal(k2[:2], kp[:2])


def test_split_partitions_recombine_to_softmax():
    rng = np.random.default_rng(19)
    L, D = 1500, 16
    keys = rng.standard_normal((L, D))
    vals = rng.standard_normal((L, D))
    qr = rng.standard_normal(D) * 3
    w = pa.attention_weights(qr, keys, 0.25)
    want = w @ vals
    for bounds in ([(0, L)], [(0, 512), (512, 1024), (1024, L)], [(0, 1), (1, 1499), (1499, L)]):
        got = pa.combine_partials(pa.partition_partials(qr, keys, vals, 0.25, bounds))
        assert np.max(np.abs(got - want)) < 1e-12
    # partition maxima really differ, so the rescale factor is exercised
    parts = pa.partition_partials(qr, keys, vals, 0.25, [(0, 10), (10, L)])
    assert parts[0][0] != parts[1][0]


def _mutants(orig):
    """Plausible slips, each planted into a copy of the oracle's attention."""
    def no_scale(q, k, s):
        return orig(q, k, 1.0)

    def neg_sign(q, k, s):
        x = -s * (k @ q)
        e = np.exp(x - x.max())
        return e / e.sum()

    def transposed(q, k, s):
        # q·K computed against the wrong axis pairing (K rows reversed)
        x = s * (k[::-1] @ q)
        e = np.exp(x - x.max())
        return e / e.sum()

    def unshifted_running_max(q, k, s):
        # the printed one-pass sketch: exp against a running max, no rescale
        x = s * (k @ q)
        m = -np.inf
        tot = 0.0
        e = np.empty_like(x)
        for i, v in enumerate(x):
            m = max(m, v)
            e[i] = math.exp(v - m)
            tot += e[i]
        return e / tot

    return {"no_scale": no_scale, "neg_sign": neg_sign, "transposed": transposed,
            "one_pass_sketch": unshifted_running_max}


def test_planted_mistakes_are_caught(monkeypatch):
    """Plant each slip in the oracle and check a pin above turns red."""
    orig = pa.attention_weights
    pins = [test_matches_brute_force_loops, test_dominant_score_selects_its_value,
            lambda: test_matches_torch_sdpa_fp64(8, 2)]
    for name, fn in _mutants(orig).items():
        monkeypatch.setattr(pa, "attention_weights", fn)
        failed = False
        for pin in pins:
            try:
                pin()
            except AssertionError:
                failed = True
                break
        assert failed, f"mutant {name} survived every pin"
        monkeypatch.setattr(pa, "attention_weights", orig)

    # wrong GQA index (h % Hkv instead of h // G) and an off-by-one gather
    def gqa_mod(q, k_pool, v_pool, tables, lens, scale, dtype, layout="NHBD"):
        B, Hq, D = q.shape
        Hkv = k_pool.shape[1]
        out = np.zeros((B, Hq, D))
        for b in range(B):
            L = int(lens[b])
            K = pa.to_f64(pa.gather_sequence(k_pool, tables[b], L, layout), dtype)
            V = pa.to_f64(pa.gather_sequence(v_pool, tables[b], L, layout), dtype)
            for h in range(Hq):
                w = orig(pa.to_f64(q, dtype)[b, h], K[:, h % Hkv], scale)
                out[b, h] = w @ V[:, h % Hkv]
        return out

    monkeypatch.setattr(pa, "paged_decode_attention", gqa_mod)
    with pytest.raises(AssertionError):
        test_gqa_groups_are_contiguous()

    real_gather = pa.gather_sequence

    def off_by_one(pool, row, L, layout="NHBD"):
        bs = pa.block_size_of(pool, layout)
        t = np.arange(int(L)) + 1
        t = np.minimum(t, len(row) * bs - 1)
        phys = np.asarray(row)[t // bs]
        return pool[phys, :, t % bs, :] if layout == "NHBD" else pool[phys, t % bs]

    monkeypatch.undo()
    monkeypatch.setattr(pa, "gather_sequence", off_by_one)
    with pytest.raises(AssertionError):
        test_matches_brute_force_loops()
    monkeypatch.setattr(pa, "gather_sequence", real_gather)
