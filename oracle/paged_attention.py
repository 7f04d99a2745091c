"""fp64 oracle for paged decode attention, KV append and block copy.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): never imported by the
product package.

What is computed (vLLM paging page, §3 phase 2): a sequence's K/V live in
fixed-size physical blocks reached through its block table; attention first
collects the blocks in table order into one logically contiguous K and V, then
runs ordinary attention — scores ``q · Kᵀ``, a softmax over them, and the
weighted sum of V.  Additions the page leaves open and that are read here
plainly:

* the scores are multiplied by ``scale`` (the page's sketch has no scale; the
  callers pass ``1/sqrt(head_dim)``);
* grouped-query attention: query head ``h`` reads KV head ``h // G`` with
  ``G = Hq / Hkv`` (contiguous groups);
* the decode query is the newest position, so every one of the ``L`` cached
  tokens is visible (no mask);
* ``L = 0`` gives an output of zeros;
* the softmax is the textbook two-pass form, ``exp(s - max s) / sum``, in
  float64.  It is NOT the one-pass "max and sum in one scan" sketch of the
  optimisation-overview page §3.2, which as printed adds ``exp(s - m)`` terms
  taken against a changing running max without rescaling the earlier ones.

Pool layouts (optimisation-overview page §3.3 gives the page shape
``[num_blocks, block_size, num_heads, head_dim]``):

* ``"NHBD"`` — ``[num_blocks, Hkv, block_size, D]`` (the library's layout);
* ``"NBHD"`` — ``[num_blocks, block_size, Hkv, D]`` (the page's layout).

Element types: pools and ``q`` arrive as raw storage — ``"f32"`` (float32),
``"f16"`` (float16) or ``"bf16"`` (uint16 bit patterns).  Widening any of them
to float64 is exact.
"""
from __future__ import annotations

import numpy as np

LAYOUTS = ("NHBD", "NBHD")
DTYPES = ("f32", "f16", "bf16", "f64")


def to_f64(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Widen raw storage to float64 exactly.

    bfloat16 is the top half of an IEEE float32, so its 16 bits shifted left by
    16 are the float32 with the same value.
    """
    if dtype == "f32":
        return np.asarray(raw, dtype=np.float32).astype(np.float64)
    if dtype == "f16":
        return np.asarray(raw, dtype=np.float16).astype(np.float64)
    if dtype == "bf16":
        bits = np.asarray(raw, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return bits.view(np.float32).astype(np.float64)
    if dtype == "f64":
        return np.asarray(raw, dtype=np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


def block_size_of(pool: np.ndarray, layout: str) -> int:
    if layout == "NHBD":
        return pool.shape[2]
    if layout == "NBHD":
        return pool.shape[1]
    raise ValueError(f"unknown layout {layout!r}")


def gather_sequence(pool: np.ndarray, table_row: np.ndarray, seq_len: int,
                    layout: str = "NHBD") -> np.ndarray:
    """Collect one sequence's cached rows in logical order → ``[L, Hkv, D]``.

    Token ``t`` sits in logical block ``t // block_size`` at offset
    ``t % block_size``; the table maps the logical block to a physical one
    (vLLM paging page §2 "page table", §3 phase 2).  Returns raw storage
    (same dtype as ``pool``).
    """
    bs = block_size_of(pool, layout)
    t = np.arange(int(seq_len))
    phys = np.asarray(table_row)[t // bs]
    off = t % bs
    if layout == "NHBD":
        return pool[phys, :, off, :]
    return pool[phys, off, :, :]


def attention_weights(q_row: np.ndarray, keys: np.ndarray, scale: float) -> np.ndarray:
    """Softmax weights of one query row over contiguous float64 keys ``[L, D]``."""
    s = scale * (keys @ q_row)
    e = np.exp(s - s.max())
    return e / e.sum()


def paged_decode_attention(q, k_pool, v_pool, block_tables, seq_lens, scale,
                           dtype: str, layout: str = "NHBD") -> np.ndarray:
    """Decode attention over a paged KV pool, float64 result ``[B, Hq, D]``.

    ``q``: ``[B, Hq, D]`` raw; pools: raw in ``layout``; ``block_tables``:
    ``[B, max_blocks]`` int; ``seq_lens``: ``[B]`` tokens already in the pool.
    """
    B, Hq, D = q.shape
    Hkv = k_pool.shape[1] if layout == "NHBD" else k_pool.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    qf = to_f64(q, dtype)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        K = to_f64(gather_sequence(k_pool, block_tables[b], L, layout), dtype)
        V = to_f64(gather_sequence(v_pool, block_tables[b], L, layout), dtype)
        for h in range(Hq):
            g = h // G
            w = attention_weights(qf[b, h], K[:, g, :], scale)
            out[b, h] = w @ V[:, g, :]
    return out


def kv_append(k_pool, v_pool, k_new, v_new, slot_mapping, layout: str = "NHBD"):
    """Write each new token's K/V rows into its slot; returns new pools.

    Slot ``s`` is physical block ``s // block_size``, offset ``s % block_size``
    (vLLM paging page §3 phase 1: the token goes into the sequence's current
    page).  ``slot < 0`` marks a padding token and writes nothing.  This is a
    copy of raw storage: the result is compared byte for byte.
    """
    bs = block_size_of(k_pool, layout)
    k_out = k_pool.copy()
    v_out = v_pool.copy()
    for i, s in enumerate(np.asarray(slot_mapping).tolist()):
        if s < 0:
            continue
        p, o = divmod(int(s), bs)
        if layout == "NHBD":
            k_out[p, :, o, :] = k_new[i]
            v_out[p, :, o, :] = v_new[i]
        else:
            k_out[p, o, :, :] = k_new[i]
            v_out[p, o, :, :] = v_new[i]
    return k_out, v_out


def copy_blocks(k_pool, v_pool, pairs):
    """Copy whole physical blocks ``src → dst`` (all heads, all offsets), in
    order; the copy-on-write step of the vLLM paging page §3 phase 3."""
    k_out = k_pool.copy()
    v_out = v_pool.copy()
    for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
        k_out[dst] = k_out[src]
        v_out[dst] = v_out[src]
    return k_out, v_out


def partition_partials(q_row, keys, values, scale, bounds):
    """Per-partition softmax statistics of one query row.

    For each token range ``[a, b)`` in ``bounds``: ``m = max s``,
    ``l = Σ exp(s - m)`` and the unnormalised ``o = Σ exp(s - m) · v``.
    """
    s = scale * (keys @ q_row)
    out = []
    for a, b in bounds:
        sp = s[a:b]
        m = sp.max()
        e = np.exp(sp - m)
        out.append((m, e.sum(), e @ values[a:b]))
    return out


def combine_partials(partials):
    """Merge per-partition ``(m, l, o)`` into the softmax-weighted output.

    With ``M = max m_p`` each partition is rescaled by ``exp(m_p - M)``:
    ``out = Σ exp(m_p - M) o_p / Σ exp(m_p - M) l_p``.  In exact arithmetic
    this equals the unsplit softmax, because every partition's terms were
    taken against its own max and the factor moves them to the common one.
    """
    M = max(m for m, _, _ in partials)
    num = sum(np.exp(m - M) * o for m, _, o in partials)
    den = sum(np.exp(m - M) * l for m, l, _ in partials)
    return num / den


def paged_prefill_attention(q, k_pool, v_pool, block_tables, seq_lens, q_lens, scale,
                            dtype: str, layout: str = "NHBD") -> np.ndarray:
    """Causal attention of a prefill chunk over a paged KV pool, float64 ``[T, Hq, D]``.

    Chunked prefill (vLLM production page §2: long prompts are fed in chunks
    and share a batch with decode steps; optimisation-overview page §2.3:
    ``enable_chunked_prefill``): sequence ``b`` brings ``n_b = q_lens[b]`` new
    query rows, packed one sequence after another in ``q`` (``T = Σ n_b``).
    Their K/V are already in the pool (written by :func:`kv_append`), so the
    pool holds ``seq_lens[b]`` tokens of which the last ``n_b`` are the
    chunk's.  Query ``i`` of the chunk sits at position
    ``p = seq_lens[b] - n_b + i`` and, causally, sees the tokens ``0 … p``
    (earlier context plus the chunk's rows up to itself).  Each row is then
    the decode computation of :func:`paged_decode_attention` over its
    visible prefix: gather through the table, scores scaled by ``scale``,
    two-pass softmax, weighted sum of V, KV head ``h // G``.
    """
    T, Hq, D = q.shape
    q_lens = [int(x) for x in np.asarray(q_lens).tolist()]
    if sum(q_lens) != T:
        raise ValueError("q rows must equal the sum of q_lens")
    Hkv = k_pool.shape[1] if layout == "NHBD" else k_pool.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    qf = to_f64(q, dtype)
    out = np.zeros((T, Hq, D), dtype=np.float64)
    row = 0
    for b, n in enumerate(q_lens):
        L = int(seq_lens[b])
        if n > L:
            raise ValueError("a chunk cannot be longer than its sequence")
        if n == 0:
            continue
        K = to_f64(gather_sequence(k_pool, block_tables[b], L, layout), dtype)
        V = to_f64(gather_sequence(v_pool, block_tables[b], L, layout), dtype)
        for i in range(n):
            p = L - n + i
            for h in range(Hq):
                g = h // G
                w = attention_weights(qf[row + i, h], K[:p + 1, g, :], scale)
                out[row + i, h] = w @ V[:p + 1, g, :]
        row += n
    return out
