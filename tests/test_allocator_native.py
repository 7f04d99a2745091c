"""The library's C++ host allocator against the Python model (CPU only).

Both sides get the same free-list order and the same operations; block ids,
slots, copy pairs, tables, lengths, statistics and error codes must agree
exactly, and the native side must satisfy the model's invariants.
"""
import json
import os

import numpy as np
import pytest

from oracle.block_allocator import AllocatorError, BlockAllocatorModel
from paged_kv_cache_406_b200 import Allocator, PagedKVError

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paging_example.json")


def _same(model: BlockAllocatorModel, nat: Allocator, ids):
    for sid in ids:
        assert nat.seq_len(sid) == model.seq_len(sid)
    if ids:
        maxb = max(len(model.block_table(s)) for s in ids) + 2
        tables, lens = nat.block_tables(list(ids), maxb)
        for i, sid in enumerate(ids):
            t = model.block_table(sid)
            assert tables[i, :len(t)].tolist() == t
            assert (tables[i, len(t):] == -1).all()
            assert lens[i] == model.seq_len(sid)
    assert nat.stats() == {**model.stats(), "block_size": model.block_size}


def test_golden_paging_example(native):
    g = json.load(open(GOLDEN))
    nat = Allocator(g["num_blocks"], g["block_size"], g["free_order"])
    nat.add(7, 0)
    slots = []
    for _ in range(g["phase1"]["tokens_appended"]):
        s, cow = nat.append_slots([7])
        assert cow.size == 0
        slots += s.tolist()
    assert slots == g["phase1"]["slots_in_order"]
    t, _ = nat.block_tables([7], 4)
    assert t[0, :2].tolist() == g["phase1"]["table_after"]
    assert nat.stats()["free_blocks"] == g["phase1"]["free_blocks_after"]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_operations_match_model(native, seed):
    rng = np.random.default_rng(seed)
    nb, bs = 97, [1, 8, 16][seed]
    order = rng.permutation(nb)
    model = BlockAllocatorModel(nb, bs, order)
    nat = Allocator(nb, bs, order)
    live, nxt = [], 0
    for _ in range(1500):
        op = int(rng.integers(0, 5))
        m_err = n_err = None
        if op == 0 or not live:
            n = int(rng.integers(0, 3 * bs + 3))
            try:
                model.add(nxt, n)
            except AllocatorError as e:
                m_err = e.code
            try:
                nat.add(nxt, n)
            except PagedKVError as e:
                n_err = e.code
            if m_err is None:
                live.append(nxt)
            nxt += 1
        elif op == 1:
            p = live[int(rng.integers(len(live)))]
            try:
                model.fork(p, nxt)
            except AllocatorError as e:
                m_err = e.code
            try:
                nat.fork(p, nxt)
            except PagedKVError as e:
                n_err = e.code
            if m_err is None:
                live.append(nxt)
            nxt += 1
        elif op in (2, 3):
            k = int(rng.integers(1, len(live) + 1))
            ids = [int(i) for i in rng.choice(live, size=k, replace=True)]  # repeats allowed
            if rng.random() < 0.05:
                ids.append(10 ** 9)  # unknown id: the whole call must be refused
            try:
                ms, mc = model.append_slots(ids)
            except AllocatorError as e:
                m_err = e.code
            try:
                ns, nc = nat.append_slots(ids)
            except PagedKVError as e:
                n_err = e.code
            if m_err is None and n_err is None:
                assert ns.tolist() == ms
                assert [tuple(x) for x in nc.tolist()] == mc
        else:
            v = live.pop(int(rng.integers(len(live))))
            model.free_seq(v)
            nat.free(v)
        assert m_err == n_err
        model.check_invariants()
        _same(model, nat, live)
    for v in live:
        model.free_seq(v)
        nat.free(v)
    assert nat.stats()["free_blocks"] == nb


@pytest.mark.parametrize("prefix,bs", [(1021, 8), (1021, 16), (1021, 32), (1024, 16)])
def test_prefix_sharing_copy_on_write(native, prefix, bs):
    n = 32
    model = BlockAllocatorModel(4000, bs)
    nat = Allocator(4000, bs)
    for a in (model, nat):
        a.add(0, prefix)
    for c in range(1, n):
        model.fork(0, c)
        nat.fork(0, c)
    ms, mc = model.append_slots(list(range(n)))
    ns, nc = nat.append_slots(list(range(n)))
    assert ns.tolist() == ms and [tuple(x) for x in nc.tolist()] == mc
    assert len(mc) == (n - 1 if prefix % bs else 0)
    assert nat.stats()["cow_copies"] == len(mc)
    _same(model, nat, list(range(n)))


def test_errors_leave_state_unchanged(native):
    nat = Allocator(3, 2)
    nat.add(0, 2)
    nat.add(1, 2)
    nat.add(2, 1)
    before = nat.stats(), nat.block_tables([0, 1, 2], 3)
    with pytest.raises(PagedKVError) as e:
        nat.append_slots([2, 0, 1])
    assert e.value.code == -2
    after = nat.stats(), nat.block_tables([0, 1, 2], 3)
    assert before[0] == after[0]
    for x, y in zip(before[1], after[1]):
        assert np.array_equal(x, y)
    with pytest.raises(PagedKVError) as e:
        nat.add(0, 1)
    assert e.value.code == -7
    with pytest.raises(PagedKVError) as e:
        nat.free(42)
    assert e.value.code == -3
    with pytest.raises(PagedKVError) as e:
        Allocator(4, 2, [0, 1, 1, 2])
    assert e.value.code == -1
    with pytest.raises(PagedKVError) as e:
        nat.block_tables([0], 0)
    assert e.value.code == -1


@pytest.mark.parametrize("seed", [3, 4])
def test_prefix_cache_matches_model(native, seed):
    """add_cached, appends, forks and frees on the C++ allocator and the model:
    identical reuse counts, tables, slots, statistics and error codes, with
    eviction of cached-free blocks when the pool runs dry."""
    rng = np.random.default_rng(seed)
    bs, nb = 4, 50
    order = rng.permutation(nb)
    model = BlockAllocatorModel(nb, bs, order)
    nat = Allocator(nb, bs, order)
    prefixes = [list(rng.integers(0, 4, size=16)) for _ in range(3)]
    live, nxt = [], 0
    for _ in range(1500):
        op = int(rng.integers(0, 5))
        m_err = n_err = m_res = n_res = None
        if op <= 1 or not live:
            toks = prefixes[int(rng.integers(3))][: int(rng.integers(0, 17))] + \
                [int(x) for x in rng.integers(0, 4, size=int(rng.integers(0, 7)))]
            try:
                m_res = model.add_cached(nxt, toks)
            except AllocatorError as e:
                m_err = e.code
            try:
                n_res = nat.add_cached(nxt, toks)
            except PagedKVError as e:
                n_err = e.code
            assert m_res == n_res
            if m_err is None:
                live.append(nxt)
            nxt += 1
        elif op == 2:
            ids = [int(x) for x in rng.choice(live, size=int(rng.integers(1, len(live) + 1)))]
            try:
                ms, mc = model.append_slots(ids)
            except AllocatorError as e:
                m_err = e.code
            try:
                ns, nc = nat.append_slots(ids)
            except PagedKVError as e:
                n_err = e.code
            if m_err is None and n_err is None:
                assert ns.tolist() == ms and [tuple(x) for x in nc.tolist()] == mc
        elif op == 3:
            p = live[int(rng.integers(len(live)))]
            model.fork(p, nxt)
            nat.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        else:
            v = live.pop(int(rng.integers(len(live))))
            model.free_seq(v)
            nat.free(v)
        assert m_err == n_err
        model.check_invariants()
        _same(model, nat, live)
    assert nat.stats()["cache_hits"] > 0
