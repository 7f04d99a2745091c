"""Pure-Python model of the host block allocator — TEST INFRASTRUCTURE ONLY.

Follows the vLLM paging page:

* §2: the cache is cut into fixed-size pages; each sequence keeps a page table
  of physical pages that need not be contiguous; the scheduler keeps a free
  page list, hands pages out when a sequence needs one and takes them back when
  it ends.
* §3 phase 1: with 8-token pages the first 8 tokens fill the first page and the
  9th token takes a new page from the free list; the table grows by one entry.
* §3 phase 3: pages of a shared prefix are not returned while another sequence
  still uses them; their reference count rises on sharing and the page is
  freed only when the last sharer ends ("copy-on-write" style sharing).
* §4: a request whose page need exceeds the free pages is refused rather than
  allocated into an out-of-memory state; aborting a request frees all of its
  pages.

Readings where the page is silent (the C++ allocator implements the same):

* the free list is a LIFO stack; ``free_order[0]`` is handed out first;
* a write into a block whose refcount is above 1 first moves the sequence to a
  fresh copy of that block (refcount of the old one drops by one) and reports
  the ``(src, dst)`` pair; sequences in one ``append_slots`` call are served in
  the order given, so of ``n`` sharers the first ``n - 1`` copy and the last
  one writes in place;
* every failing call leaves the state exactly as it was (all-or-nothing);
* a freed sequence returns its blocks in table order, so its last block ends
  on top of the stack.

Prefix caching (vLLM paging page §3 phase 3 and §5 "enable_prefix_caching";
vLLM production page §5: reusing blocks costs hashing time and helps only
repeated prefixes) — readings taken:

* a *full* block admitted with known token ids is identified by the token ids
  of the whole prefix up to and including it (the chain of its predecessors);
  a sequence admitted with ``add_cached`` reuses the longest run of leading
  full blocks whose identities are cached (refcount + 1) and takes fresh blocks
  for the rest; its partial last block is always fresh;
* fresh full blocks of an ``add_cached`` admission are registered under their
  identity unless that identity is already registered (a later block of a
  prefix can outlive an evicted earlier one); blocks filled later by appends
  are not registered;
* a registered block whose refcount drops to zero stays registered as
  *cached-free*: a later hit revives it; it is evicted (unregistered and handed
  out) only when the free stack is empty, least recently freed first;
* a registered block is never written (appends go to partial blocks, which are
  never registered).
"""
from __future__ import annotations

import copy

OK = 0
ERR_INVALID_ARG = -1
ERR_OUT_OF_BLOCKS = -2
ERR_UNKNOWN_SEQ = -3
ERR_SEQ_EXISTS = -7


class AllocatorError(Exception):
    def __init__(self, code: int, msg: str):
        super().__init__(msg)
        self.code = code


class BlockAllocatorModel:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise AllocatorError(ERR_INVALID_ARG, "sizes must be positive")
        order = list(range(num_blocks)) if free_order is None else [int(x) for x in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise AllocatorError(ERR_INVALID_ARG, "free_order is not a permutation")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = list(reversed(order))  # top of stack = end of list
        self.refcount = [0] * num_blocks
        self.seqs: dict[int, list] = {}  # id -> [table, length]
        self.cow_copies = 0
        self.cache: dict[tuple, int] = {}  # prefix token tuple -> block
        self.block_key: dict[int, tuple] = {}
        self.lru: list[int] = []           # cached-free blocks, least recently freed first
        self.cache_queries = 0
        self.cache_hits = 0

    # -- helpers --------------------------------------------------------
    def _pop(self) -> int:
        if self.free:
            b = self.free.pop()
        elif self.lru:  # evict the least recently freed cached block
            b = self.lru.pop(0)
            del self.cache[self.block_key.pop(b)]
        else:
            raise AllocatorError(ERR_OUT_OF_BLOCKS, "no free block")
        self.refcount[b] = 1
        return b

    def _available(self) -> int:
        return len(self.free) + len(self.lru)

    def _state(self):
        return (self.free, self.refcount, self.seqs, self.cow_copies, self.cache, self.block_key, self.lru,
                self.cache_queries, self.cache_hits)

    def _atomic(self, fn):
        saved = copy.deepcopy(self._state())
        try:
            return fn()
        except AllocatorError:
            (self.free, self.refcount, self.seqs, self.cow_copies, self.cache, self.block_key, self.lru,
             self.cache_queries, self.cache_hits) = saved
            raise

    # -- operations ------------------------------------------------------
    def add(self, seq_id: int, n_tokens: int) -> None:
        if n_tokens < 0:
            raise AllocatorError(ERR_INVALID_ARG, "negative length")
        if seq_id in self.seqs:
            raise AllocatorError(ERR_SEQ_EXISTS, "sequence exists")
        need = -(-n_tokens // self.block_size)
        if need > self._available():
            raise AllocatorError(ERR_OUT_OF_BLOCKS, "admission refused")
        table = [self._pop() for _ in range(need)]
        self.seqs[seq_id] = [table, n_tokens]

    def add_cached(self, seq_id: int, tokens) -> int:
        """Admit a sequence holding ``tokens``, reusing cached full blocks of its
        prefix; returns the number of leading tokens whose blocks were reused."""
        tokens = [int(t) for t in tokens]
        if seq_id in self.seqs:
            raise AllocatorError(ERR_SEQ_EXISTS, "sequence exists")
        bs = self.block_size
        n = len(tokens)
        nfull = n // bs
        hits = 0
        while hits < nfull and tuple(tokens[:(hits + 1) * bs]) in self.cache:
            hits += 1
        need = -(-n // bs) - hits
        # revived cached-free blocks leave the evictable set, so they do not count as available
        revived = sum(1 for i in range(hits) if self.refcount[self.cache[tuple(tokens[:(i + 1) * bs])]] == 0)
        if need > self._available() - revived:
            raise AllocatorError(ERR_OUT_OF_BLOCKS, "admission refused")
        self.cache_queries += nfull
        self.cache_hits += hits
        table = []
        for i in range(hits):
            b = self.cache[tuple(tokens[:(i + 1) * bs])]
            if self.refcount[b] == 0:
                self.lru.remove(b)
            self.refcount[b] += 1
            table.append(b)
        for i in range(hits, -(-n // bs)):
            b = self._pop()
            table.append(b)
            key = tuple(tokens[:(i + 1) * bs])
            if i < nfull and key not in self.cache:  # a later block may still be cached after an eviction
                self.cache[key] = b
                self.block_key[b] = key
        self.seqs[seq_id] = [table, n]
        return hits * bs

    def fork(self, parent: int, child: int) -> None:
        if parent not in self.seqs:
            raise AllocatorError(ERR_UNKNOWN_SEQ, "unknown parent")
        if child in self.seqs:
            raise AllocatorError(ERR_SEQ_EXISTS, "child exists")
        table, n = self.seqs[parent]
        for b in table:
            self.refcount[b] += 1
        self.seqs[child] = [list(table), n]

    def append_slots(self, seq_ids):
        """Reserve one slot per listed sequence; returns ``(slots, cow_pairs)``."""
        def run():
            slots, cows = [], []
            for sid in seq_ids:
                if sid not in self.seqs:
                    raise AllocatorError(ERR_UNKNOWN_SEQ, f"unknown sequence {sid}")
                entry = self.seqs[sid]
                table, pos = entry
                bi, off = divmod(pos, self.block_size)
                if off == 0:
                    table.append(self._pop())
                else:
                    old = table[bi]
                    if self.refcount[old] > 1:
                        new = self._pop()
                        self.refcount[old] -= 1
                        table[bi] = new
                        cows.append((old, new))
                        self.cow_copies += 1
                slots.append(table[bi] * self.block_size + off)
                entry[1] = pos + 1
            return slots, cows
        return self._atomic(run)

    def free_seq(self, seq_id: int) -> None:
        if seq_id not in self.seqs:
            raise AllocatorError(ERR_UNKNOWN_SEQ, "unknown sequence")
        table, _ = self.seqs.pop(seq_id)
        for b in table:
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                if b in self.block_key:
                    self.lru.append(b)  # stays cached until evicted
                else:
                    self.free.append(b)

    def block_table(self, seq_id: int) -> list:
        return list(self.seqs[seq_id][0])

    def seq_len(self, seq_id: int) -> int:
        return self.seqs[seq_id][1]

    def stats(self) -> dict:
        fill = {}
        for table, n in self.seqs.values():
            for i, b in enumerate(table):
                used = min(self.block_size, n - i * self.block_size)
                fill[b] = max(fill.get(b, 0), used)
        return {
            "num_blocks": self.num_blocks,
            "free_blocks": len(self.free) + len(self.lru),
            "used_blocks": self.num_blocks - len(self.free) - len(self.lru),
            "num_seqs": len(self.seqs),
            "cow_copies": self.cow_copies,
            "logical_tokens": sum(n for _, n in self.seqs.values()),
            "waste_tokens": sum(self.block_size - f for f in fill.values()),
            "cached_blocks": len(self.block_key),
            "cache_queries": self.cache_queries,
            "cache_hits": self.cache_hits,
        }

    def check_invariants(self) -> None:
        """The bookkeeping identities every state must satisfy."""
        count = [0] * self.num_blocks
        for table, n in self.seqs.values():
            assert len(table) == -(-n // self.block_size)
            for b in set(table):
                count[b] += table.count(b)
        assert count == self.refcount, "refcount != number of tables holding the block"
        free = set(self.free)
        lru = set(self.lru)
        assert len(free) == len(self.free), "block twice on the free list"
        assert len(lru) == len(self.lru), "block twice on the cached-free list"
        assert not free & lru
        for b in range(self.num_blocks):
            assert (self.refcount[b] == 0) == (b in free or b in lru)
        assert lru <= set(self.block_key), "cached-free blocks are registered"
        assert not free & set(self.block_key), "stack blocks are not registered"
        assert all(self.cache[k] == b for b, k in self.block_key.items())
        used = sum(1 for r in self.refcount if r > 0)
        assert used + len(self.free) + len(self.lru) == self.num_blocks
