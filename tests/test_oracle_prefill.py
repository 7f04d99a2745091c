"""Pins for the fp64 causal chunked-prefill oracle (CPU only).

``paged_prefill_attention`` is tied to things other than itself: PyTorch's CPU
scaled-dot-product attention in float64 (its ``is_causal`` lower-triangular
mask for a whole prompt, an explicit boolean mask for a chunk behind earlier
context), explicit Python loops on a tiny case, the decode oracle (a chunk of
one row is a decode query), closed forms (the first position returns its own
V row; constant V), and invariants (a chunk split into smaller chunks gives
the same rows; any permutation of physical blocks or block size).  A mask
shifted by one, a mask pointing the wrong way, a query position that ignores
the earlier context, or rows packed in the wrong order each fail one of them;
``test_planted_mistakes_are_caught`` plants each in the oracle.
"""
import math

import numpy as np
import pytest
import torch

from oracle import paged_attention as pa
from test_oracle import _scatter


def _case(rng, lens, q_lens, Hq, Hkv, D, dtype=np.float32):
    Ks = [rng.standard_normal((L, Hkv, D)).astype(dtype) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D)).astype(dtype) for L in lens]
    q = rng.standard_normal((sum(q_lens), Hq, D)).astype(dtype)
    return q, Ks, Vs


def _paged(q, Ks, Vs, q_lens, scale, bs, perm_seed, layout="NHBD"):
    lens = [len(k) for k in Ks]
    nb = sum(-(-L // bs) for L in lens)
    perm = np.random.default_rng(perm_seed).permutation(max(nb, 1))
    kp, tables = _scatter(Ks, bs, perm, layout)
    vp, _ = _scatter(Vs, bs, perm, layout)
    return pa.paged_prefill_attention(q, kp, vp, tables, np.array(lens), np.array(q_lens), scale, "f32", layout)


def _sdpa(q_rows, K, V, scale, G, ctx):
    """torch SDPA in float64 for one sequence: rows ``[n, Hq, D]`` at positions
    ``ctx .. ctx+n-1`` over contiguous ``K, V`` of ``[L, Hkv, D]``."""
    qt = torch.from_numpy(q_rows.astype(np.float64)).permute(1, 0, 2)            # [Hq, n, D]
    kt = torch.from_numpy(K.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    vt = torch.from_numpy(V.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    n, L = q_rows.shape[0], K.shape[0]
    if ctx == 0 and n == L:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    else:
        mask = torch.arange(L)[None, :] <= (ctx + torch.arange(n))[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (32, 8)])
def test_whole_prompts_match_torch_causal_sdpa(Hq, Hkv):
    rng = np.random.default_rng(11)
    lens = [1, 5, 37, 64]
    D, scale = 16, 0.29
    q, Ks, Vs = _case(rng, lens, lens, Hq, Hkv, D)
    got = _paged(q, Ks, Vs, lens, scale, bs=16, perm_seed=12)
    row = 0
    for b, L in enumerate(lens):
        want = _sdpa(q[row:row + L], Ks[b], Vs[b], scale, Hq // Hkv, 0)
        assert np.max(np.abs(got[row:row + L] - want)) < 1e-12
        row += L


def test_chunks_behind_context_match_masked_sdpa():
    rng = np.random.default_rng(13)
    lens, q_lens = [40, 100, 7, 130], [9, 1, 7, 64]
    Hq, Hkv, D, scale = 8, 2, 16, 1 / math.sqrt(16)
    q, Ks, Vs = _case(rng, lens, q_lens, Hq, Hkv, D)
    got = _paged(q, Ks, Vs, q_lens, scale, bs=8, perm_seed=14)
    row = 0
    for b, (L, n) in enumerate(zip(lens, q_lens)):
        want = _sdpa(q[row:row + n], Ks[b], Vs[b], scale, Hq // Hkv, L - n)
        assert np.max(np.abs(got[row:row + n] - want)) < 1e-12
        row += n


def test_tiny_case_matches_explicit_loops():
    rng = np.random.default_rng(15)
    lens, q_lens = [6, 3], [4, 3]
    Hq, Hkv, D, scale = 2, 1, 3, 0.8
    q, Ks, Vs = _case(rng, lens, q_lens, Hq, Hkv, D)
    got = _paged(q, Ks, Vs, q_lens, scale, bs=2, perm_seed=16)
    row = 0
    for b, (L, n) in enumerate(zip(lens, q_lens)):
        for i in range(n):
            pos = L - n + i
            for h in range(Hq):
                s = [scale * sum(float(q[row + i, h, d]) * float(Ks[b][t, 0, d]) for d in range(D))
                     for t in range(pos + 1)]
                mx = max(s)
                e = [math.exp(x - mx) for x in s]
                for d in range(D):
                    want = sum(e[t] * float(Vs[b][t, 0, d]) for t in range(pos + 1)) / sum(e)
                    assert abs(got[row + i, h, d] - want) < 1e-12
        row += n


def test_one_row_chunks_are_decode_queries():
    rng = np.random.default_rng(17)
    lens = [1, 16, 17, 50]
    q, Ks, Vs = _case(rng, lens, [1] * 4, 8, 2, 16)
    got = _paged(q, Ks, Vs, [1] * 4, 0.25, bs=16, perm_seed=18)
    perm = np.random.default_rng(18).permutation(sum(-(-L // 16) for L in lens))
    kp, tables = _scatter(Ks, 16, perm)
    vp, _ = _scatter(Vs, 16, perm)
    want = pa.paged_decode_attention(q, kp, vp, tables, np.array(lens), 0.25, "f32")
    assert np.max(np.abs(got - want)) < 1e-12


def test_closed_forms_first_position_and_constant_v():
    rng = np.random.default_rng(19)
    lens = [5, 33]
    q, Ks, Vs = _case(rng, lens, lens, 4, 2, 8)
    got = _paged(q, Ks, Vs, lens, 0.5, bs=4, perm_seed=20)
    # position 0 sees only itself: the output is its V row, exactly
    assert np.array_equal(got[0], np.repeat(Vs[0][0].astype(np.float64), 2, axis=0))
    assert np.array_equal(got[5], np.repeat(Vs[1][0].astype(np.float64), 2, axis=0))
    Vc = [np.full_like(v, 0.75) for v in Vs]
    got = _paged(q, Ks, Vc, lens, 0.5, bs=4, perm_seed=20)
    assert np.max(np.abs(got - 0.75)) < 1e-15


def test_splitting_a_chunk_gives_the_same_rows():
    """Chunked prefill: rows computed in several smaller chunks (each call
    seeing only the context written so far) equal the one-shot rows."""
    rng = np.random.default_rng(21)
    L, Hq, Hkv, D, scale, bs = 70, 4, 2, 8, 0.35, 8
    q, Ks, Vs = _case(rng, [L], [L], Hq, Hkv, D)
    whole = _paged(q, Ks, Vs, [L], scale, bs, perm_seed=22)
    parts, start = [], 0
    for n in (13, 1, 40, 16):
        end = start + n
        parts.append(_paged(q[start:end], [Ks[0][:end]], [Vs[0][:end]], [n], scale, bs, perm_seed=23 + start))
        start = end
    assert np.max(np.abs(np.concatenate(parts) - whole)) < 1e-12


@pytest.mark.parametrize("bs,layout", [(1, "NHBD"), (8, "NBHD"), (32, "NHBD")])
def test_block_size_permutation_and_layout_invariance(bs, layout):
    rng = np.random.default_rng(25)
    lens, q_lens = [45, 9], [20, 9]
    q, Ks, Vs = _case(rng, lens, q_lens, 4, 4, 8)
    ref = _paged(q, Ks, Vs, q_lens, 0.3, bs=16, perm_seed=26)
    got = _paged(q, Ks, Vs, q_lens, 0.3, bs=bs, perm_seed=27, layout=layout)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_argument_checks_and_empty_chunks():
    rng = np.random.default_rng(29)
    q, Ks, Vs = _case(rng, [4, 6], [0, 2], 2, 2, 4)
    got = _paged(q, Ks, Vs, [0, 2], 1.0, bs=4, perm_seed=30)
    assert got.shape == (2, 2, 4)
    kp, tables = _scatter(Ks, 4, np.arange(3))
    with pytest.raises(ValueError):
        pa.paged_prefill_attention(q, kp, kp, tables, np.array([4, 1]), np.array([0, 2]), 1.0, "f32")
    with pytest.raises(ValueError):
        pa.paged_prefill_attention(q, kp, kp, tables, np.array([4, 6]), np.array([1, 2]), 1.0, "f32")


def test_planted_mistakes_are_caught(monkeypatch):
    """Plant each slip in the oracle's position or mask logic and check that
    a pin above turns red."""
    real = pa.paged_prefill_attention

    def variant(kind):
        def fn(q, k_pool, v_pool, tables, seq_lens, q_lens, scale, dtype, layout="NHBD"):
            Hq = q.shape[1]
            Hkv = k_pool.shape[1] if layout == "NHBD" else k_pool.shape[2]
            G = Hq // Hkv
            qf = pa.to_f64(q, dtype)
            out = np.zeros(q.shape, dtype=np.float64)
            row = 0
            for b, n in enumerate(np.asarray(q_lens).tolist()):
                L = int(seq_lens[b])
                if n > L or n == 0:
                    continue
                K = pa.to_f64(pa.gather_sequence(k_pool, tables[b], L, layout), dtype)
                V = pa.to_f64(pa.gather_sequence(v_pool, tables[b], L, layout), dtype)
                for i in range(n):
                    p = {"no_context": i, "mask_short": L - n + i - 1, "mask_long": L - n + i + 1}.get(kind, L - n + i)
                    p = max(0, min(p, L - 1))
                    sel = slice(p, L) if kind == "reversed" else slice(0, p + 1)
                    r = (row + n - 1 - i) if kind == "row_order" else row + i
                    for h in range(Hq):
                        w = pa.attention_weights(qf[r, h], K[sel, h // G], scale)
                        out[row + i, h] = w @ V[sel, h // G]
                row += n
            return out
        return fn

    pins = [lambda: test_whole_prompts_match_torch_causal_sdpa(8, 2), test_chunks_behind_context_match_masked_sdpa,
            test_one_row_chunks_are_decode_queries, test_closed_forms_first_position_and_constant_v]
    monkeypatch.setattr(pa, "paged_prefill_attention", variant("exact"))  # the harness itself is sound
    for pin in pins:
        pin()
    for kind in ("no_context", "mask_short", "mask_long", "reversed", "row_order"):
        monkeypatch.setattr(pa, "paged_prefill_attention", variant(kind))
        failed = False
        for pin in pins:
            try:
                pin()
            except AssertionError:
                failed = True
                break
        assert failed, f"planted mistake {kind} survived every pin"
    monkeypatch.setattr(pa, "paged_prefill_attention", real)
    test_chunks_behind_context_match_masked_sdpa()
