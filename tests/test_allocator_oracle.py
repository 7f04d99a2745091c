"""Pins for the Python block-allocator model (CPU only).

Pinned by the worked paging example of the vLLM paging page (§3 phases 1 and
3, stored in ``tests/golden/paging_example.json``), by closed-form block counts
(``ceil(n / block_size)`` blocks per sequence, ``n - 1`` copies when ``n``
sharers each append into a shared partial block; for prefix caching the
number of reused blocks, the prefix property, revival and eviction order, and
blocks used by a shared system prompt), and by the bookkeeping invariants
checked after every operation of seeded random workloads.
"""
import json
import os

import numpy as np
import pytest

from oracle.block_allocator import (ERR_OUT_OF_BLOCKS, ERR_SEQ_EXISTS, ERR_UNKNOWN_SEQ,
                                    AllocatorError, BlockAllocatorModel)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paging_example.json")


def test_paging_page_worked_example_phase1():
    g = json.load(open(GOLDEN))
    a = BlockAllocatorModel(g["num_blocks"], g["block_size"], g["free_order"])
    a.add(7, 0)
    lens, slots = [], []
    for _ in range(g["phase1"]["tokens_appended"]):
        s, cow = a.append_slots([7])
        assert cow == []
        slots += s
        lens.append(len(a.block_table(7)))
        a.check_invariants()
    assert lens == g["phase1"]["table_len_after_each_token"]
    assert a.block_table(7) == g["phase1"]["table_after"]
    assert slots == g["phase1"]["slots_in_order"]
    assert a.stats()["free_blocks"] == g["phase1"]["free_blocks_after"]


def test_paging_page_worked_example_phase3():
    g = json.load(open(GOLDEN))
    a = BlockAllocatorModel(g["num_blocks"], g["block_size"], g["free_order"])
    a.add(1, g["phase3"]["shared_prefix_tokens"])
    for c in range(2, g["phase3"]["sharers"] + 1):
        a.fork(1, c)
    a.check_invariants()
    a.free_seq(1)
    a.check_invariants()
    assert a.stats()["free_blocks"] == g["phase3"]["free_blocks_after_first_sharer_ends"]
    for c in range(2, g["phase3"]["sharers"] + 1):
        a.free_seq(c)
    assert a.stats()["free_blocks"] == g["phase3"]["free_blocks_after_last_sharer_ends"]
    a.check_invariants()


@pytest.mark.parametrize("bs", [1, 8, 16, 32])
def test_blocks_per_sequence_is_ceil(bs):
    a = BlockAllocatorModel(1000, bs)
    for i, n in enumerate([0, 1, bs - 1, bs, bs + 1, 3 * bs + 2]):
        a.add(i, n)
        assert len(a.block_table(i)) == -(-n // bs)
    a.check_invariants()


def test_admission_refused_without_change():
    a = BlockAllocatorModel(4, 16)
    a.add(0, 40)  # 3 blocks
    before = (list(a.free), list(a.refcount), a.stats())
    with pytest.raises(AllocatorError) as e:
        a.add(1, 17)  # needs 2, only 1 free
    assert e.value.code == ERR_OUT_OF_BLOCKS
    assert (list(a.free), list(a.refcount), a.stats()) == before
    assert 1 not in a.seqs


def test_append_all_or_nothing():
    a = BlockAllocatorModel(3, 2)
    a.add(0, 2)
    a.add(1, 2)
    a.add(2, 1)
    before = (list(a.free), list(a.refcount), {k: (list(v[0]), v[1]) for k, v in a.seqs.items()})
    # seq 2 fits in place; seqs 0 and 1 need a block each but only 0 free
    with pytest.raises(AllocatorError) as e:
        a.append_slots([2, 0, 1])
    assert e.value.code == ERR_OUT_OF_BLOCKS
    after = (list(a.free), list(a.refcount), {k: (list(v[0]), v[1]) for k, v in a.seqs.items()})
    assert after == before
    with pytest.raises(AllocatorError) as e:
        a.append_slots([2, 99])
    assert e.value.code == ERR_UNKNOWN_SEQ
    assert a.seq_len(2) == 1


def test_errors():
    a = BlockAllocatorModel(8, 4)
    a.add(0, 3)
    with pytest.raises(AllocatorError) as e:
        a.add(0, 1)
    assert e.value.code == ERR_SEQ_EXISTS
    with pytest.raises(AllocatorError) as e:
        a.fork(5, 6)
    assert e.value.code == ERR_UNKNOWN_SEQ
    with pytest.raises(AllocatorError) as e:
        a.fork(0, 0)
    assert e.value.code == ERR_SEQ_EXISTS
    a.free_seq(0)
    with pytest.raises(AllocatorError) as e:
        a.free_seq(0)
    assert e.value.code == ERR_UNKNOWN_SEQ


@pytest.mark.parametrize("prefix,bs", [(1021, 8), (1021, 16), (1021, 32), (1024, 16)])
def test_shared_partial_block_copies_n_minus_1(prefix, bs):
    n = 32
    a = BlockAllocatorModel(2000, bs)
    a.add(0, prefix)
    for c in range(1, n):
        a.fork(0, c)
    slots, cows = a.append_slots(list(range(n)))
    partial = prefix % bs != 0
    assert len(cows) == (n - 1 if partial else 0)
    assert len(set(slots)) == n
    if partial:
        shared = a.block_table(n - 1)[-1]
        # the last sharer keeps the original block and writes in place
        assert all(src == shared for src, _ in cows)
        assert a.refcount[shared] == 1
    a.check_invariants()


def test_random_workload_keeps_invariants_and_frees_everything():
    rng = np.random.default_rng(406)
    a = BlockAllocatorModel(200, 8, rng.permutation(200))
    live = []
    nxt = 0
    for _ in range(3000):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                a.add(nxt, int(rng.integers(0, 40)))
                live.append(nxt)
                nxt += 1
            elif op == 1:
                p = live[int(rng.integers(len(live)))]
                a.fork(p, nxt)
                live.append(nxt)
                nxt += 1
            elif op == 2:
                k = int(rng.integers(1, len(live) + 1))
                ids = list(rng.choice(live, size=k, replace=False))
                a.append_slots([int(i) for i in ids])
            else:
                v = live.pop(int(rng.integers(len(live))))
                a.free_seq(v)
        except AllocatorError as e:
            assert e.code == ERR_OUT_OF_BLOCKS
        a.check_invariants()
    for v in live:
        a.free_seq(v)
    a.check_invariants()
    assert a.stats()["free_blocks"] == 200


def test_waste_accounting():
    a = BlockAllocatorModel(10, 16)
    a.add(0, 17)  # 2 blocks, 15 empty slots
    a.add(1, 32)  # full
    assert a.stats()["waste_tokens"] == 15
    a.fork(0, 2)  # shared blocks counted once
    assert a.stats()["waste_tokens"] == 15
    assert a.stats()["logical_tokens"] == 17 + 32 + 17


# ---------------------------------------------------------------------------
# prefix caching (vLLM paging page §3 phase 3, §5; vLLM production page §5)
# ---------------------------------------------------------------------------

def test_prefix_cache_reuses_full_blocks_of_identical_prefix():
    bs = 4
    a = BlockAllocatorModel(64, bs)
    toks = list(range(100, 114))  # 14 tokens: 3 full blocks + 2
    assert a.add_cached(0, toks) == 0
    assert a.add_cached(1, toks) == 12  # the 3 full blocks, never the partial one
    t0, t1 = a.block_table(0), a.block_table(1)
    assert t1[:3] == t0[:3] and t1[3] != t0[3]
    assert all(a.refcount[b] == 2 for b in t0[:3])
    st = a.stats()
    assert (st["cache_queries"], st["cache_hits"], st["cached_blocks"]) == (6, 3, 3)
    a.check_invariants()


def test_prefix_cache_stops_at_first_difference():
    bs = 4
    a = BlockAllocatorModel(64, bs)
    base = list(range(16))
    a.add_cached(0, base)
    other = base[:4] + [99] + base[5:]  # differs inside block 1
    assert a.add_cached(1, other) == 4
    assert a.block_table(1)[0] == a.block_table(0)[0]
    assert a.block_table(1)[1:] != a.block_table(0)[1:]
    # a prefix of a block is not a hit: 3 tokens of block 0 only
    assert a.add_cached(2, base[:3]) == 0
    a.check_invariants()


def test_cached_blocks_survive_free_and_are_revived():
    bs = 4
    a = BlockAllocatorModel(16, bs)
    toks = list(range(8))
    a.add_cached(0, toks)
    t0 = a.block_table(0)
    a.free_seq(0)
    st = a.stats()
    assert st["free_blocks"] == 16 and st["cached_blocks"] == 2  # free to use, still cached
    assert a.add_cached(1, toks) == 8
    assert a.block_table(1) == t0
    a.check_invariants()


def test_cached_free_blocks_are_evicted_least_recently_freed_first():
    bs = 2
    a = BlockAllocatorModel(4, bs, free_order=[0, 1, 2, 3])
    a.add_cached(0, [1, 2])      # block 0
    a.add_cached(1, [3, 4])      # block 1
    a.free_seq(1)                # freed first
    a.free_seq(0)
    a.add(2, 4)                  # takes the two stack blocks 2, 3
    assert a.block_table(2) == [2, 3]
    a.add(3, 2)                  # stack empty: evicts block 1 (freed first)
    assert a.block_table(3) == [1]
    assert a.add_cached(5, [1, 2]) == 2   # block 0 is still cached-free: revived, no new block
    assert a.block_table(5) == [0]
    with pytest.raises(AllocatorError) as e:  # [3, 4] was evicted with block 1 and the pool is full
        a.add_cached(4, [3, 4])
    assert e.value.code == ERR_OUT_OF_BLOCKS
    a.check_invariants()


def test_prefix_cache_eviction_then_readmission_consistent():
    bs = 2
    a = BlockAllocatorModel(4, bs, free_order=[0, 1, 2, 3])
    a.add_cached(0, [1, 2, 3, 4])  # blocks 0 (prefix [1,2]), 1 (prefix [1,2,3,4])
    a.free_seq(0)                  # both cached-free: 0 then 1
    a.add(1, 4)                    # stack blocks 2, 3
    a.add(2, 2)                    # evicts block 0: the first prefix block
    # [1,2] is gone but [1,2,3,4] is still cached: no hit (the chain starts with a miss)
    a.free_seq(2)
    assert a.add_cached(3, [1, 2, 3, 4]) == 0
    a.check_invariants()


def test_system_prompt_blocks_counted_once():
    """32 requests with a shared 1024-token system prompt and distinct
    100-token questions, admitted with prefix caching: the pool holds the
    prompt once plus each request's own blocks."""
    bs, n, prompt = 16, 32, 1024
    a = BlockAllocatorModel(4000, bs)
    rng = np.random.default_rng(3)
    sys_prompt = list(rng.integers(0, 32000, size=prompt))
    reused = [a.add_cached(i, sys_prompt + list(rng.integers(0, 32000, size=100))) for i in range(n)]
    assert reused == [0] + [prompt] * (n - 1)
    own = -(-(prompt + 100) // bs) - prompt // bs
    assert a.stats()["used_blocks"] == prompt // bs + n * own
    a.check_invariants()


def test_random_workload_with_prefix_cache_keeps_invariants():
    rng = np.random.default_rng(77)
    bs = 4
    a = BlockAllocatorModel(60, bs, rng.permutation(60))
    prefixes = [list(rng.integers(0, 5, size=12)) for _ in range(3)]
    live, nxt = [], 0
    for _ in range(2000):
        op = int(rng.integers(0, 5))
        try:
            if op <= 1 or not live:
                toks = prefixes[int(rng.integers(3))][: int(rng.integers(0, 13))] + \
                    list(rng.integers(0, 5, size=int(rng.integers(0, 6))))
                a.add_cached(nxt, toks)
                live.append(nxt)
                nxt += 1
            elif op == 2:
                a.append_slots([int(x) for x in rng.choice(live, size=int(rng.integers(1, len(live) + 1)))])
            elif op == 3:
                a.fork(live[int(rng.integers(len(live)))], nxt)
                live.append(nxt)
                nxt += 1
            else:
                a.free_seq(live.pop(int(rng.integers(len(live)))))
        except AllocatorError as e:
            assert e.code == ERR_OUT_OF_BLOCKS
        a.check_invariants()
