// Host-side block allocator: free stack, per-block reference counts,
// copy-on-write on a write into a shared block, all-or-nothing errors.
//
// Follows "vLLM's 'memory paging' — PagedAttention illustrated":
//   §2        fixed-size pages, a page table per sequence, a free page list;
//   §3 ph. 1  the token after a full page takes a new page, the table grows;
//   §3 ph. 3  shared prefix pages carry a reference count and are reclaimed
//             by the last sharer ("copy-on-write" style sharing);
//   §4        admission refuses requests that do not fit; abort frees pages.
//   §5 / production page §5  prefix caching: full blocks admitted with their
//             token ids are indexed by a hash of the whole prefix; a later
//             admission with the same leading tokens reuses them.
// Every operation is O(1) per token (O(blocks) for free/fork/tables); none
// touches the GPU.
//
// Prefix-cache readings (the pages name the feature, not its rules): a block
// is reused only for an identical token prefix (64-bit FNV-1a chain hash,
// verified against the stored tokens and parent hash on every hit); the
// longest run of leading full blocks is reused; a registered block whose
// refcount reaches zero stays indexed ("cached-free") until it is revived by
// a hit or evicted, least recently freed first, when the free stack is empty.
#include <algorithm>
#include <cstdint>
#include <unordered_map>
#include <vector>

#include "pkv_internal.h"

using pkv::fail;

namespace {

struct Seq {
  std::vector<int32_t> table;  // logical block -> physical block
  int32_t len = 0;             // tokens held
};

// One reversible mutation made by pkv_seq_append_slots.
struct Undo {
  enum Kind { kPop, kPopEvicted, kTablePush, kTableSet, kRefDec, kLen, kCow } kind;
  Seq* seq;
  int32_t a;  // block id, table index or old length
  int32_t b;  // old table value
};

constexpr uint64_t kFnvBasis = 14695981039346656037ull;  // FNV-1a 64-bit offset basis
constexpr uint64_t kFnvPrime = 1099511628211ull;

// FNV-1a over 32-bit token ids (one xor-multiply step per token rather than
// per byte).  Identities are verified against the stored tokens, so the hash
// only has to spread keys, not to be collision-free.
uint64_t fnv1a(uint64_t h, const int32_t* tokens, size_t n) {
  for (size_t i = 0; i < n; ++i) {
    h ^= static_cast<uint32_t>(tokens[i]);
    h *= kFnvPrime;
  }
  return h;
}

// Prefix-cache state of one physical block.
struct BlockMeta {
  bool registered = false;  // indexed under `key`
  bool in_lru = false;      // registered with refcount 0
  int32_t prev = -1, next = -1;  // cached-free list links
  uint64_t key = 0, parent = 0;  // chain hash of the prefix through this block, and of the one before it
};

}  // namespace

struct pkv_alloc {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> free_stack;  // back() is handed out next
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, Seq> seqs;
  int64_t cow_copies = 0;
  std::vector<Undo> undo;  // scratch for append_slots
  // prefix cache
  std::vector<BlockMeta> meta;
  std::vector<int32_t> block_tokens;  // [num_blocks][block_size], filled when a block is registered
  std::unordered_map<uint64_t, int32_t> cache;  // chain hash -> block
  int32_t lru_head = -1, lru_tail = -1, lru_size = 0;
  int64_t cache_queries = 0, cache_hits = 0;

  int64_t available() const { return static_cast<int64_t>(free_stack.size()) + lru_size; }

  void lru_remove(int32_t b) {
    BlockMeta& m = meta[b];
    if (m.prev >= 0) meta[m.prev].next = m.next; else lru_head = m.next;
    if (m.next >= 0) meta[m.next].prev = m.prev; else lru_tail = m.prev;
    m.prev = m.next = -1;
    m.in_lru = false;
    --lru_size;
  }
  void lru_push_back(int32_t b) {
    BlockMeta& m = meta[b];
    m.prev = lru_tail;
    m.next = -1;
    if (lru_tail >= 0) meta[lru_tail].next = b; else lru_head = b;
    lru_tail = b;
    m.in_lru = true;
    ++lru_size;
  }
  void lru_push_front(int32_t b) {
    BlockMeta& m = meta[b];
    m.prev = -1;
    m.next = lru_head;
    if (lru_head >= 0) meta[lru_head].prev = b; else lru_tail = b;
    lru_head = b;
    m.in_lru = true;
    ++lru_size;
  }

  // Hands out a block: the free stack first, else the least recently freed
  // cached block (unregistered).  *evicted tells which.  Caller checked
  // available() > 0.
  int32_t pop(bool* evicted = nullptr) {
    int32_t b;
    if (!free_stack.empty()) {
      b = free_stack.back();
      free_stack.pop_back();
      if (evicted) *evicted = false;
    } else {
      b = lru_head;
      lru_remove(b);
      cache.erase(meta[b].key);
      meta[b].registered = false;
      if (evicted) *evicted = true;
    }
    refcount[b] = 1;
    return b;
  }

  // Returns a block whose refcount reached zero.
  void release(int32_t b) {
    if (meta[b].registered) lru_push_back(b);
    else free_stack.push_back(b);
  }

  // Block holding exactly this prefix (hash h, parent hash, tokens), or -1.
  int32_t lookup(uint64_t h, uint64_t parent, const int32_t* toks) const {
    auto it = cache.find(h);
    if (it == cache.end()) return -1;
    const int32_t b = it->second;
    if (meta[b].parent != parent) return -1;
    if (!std::equal(toks, toks + block_size, block_tokens.begin() + static_cast<int64_t>(b) * block_size)) return -1;
    return b;
  }
};

extern "C" int pkv_alloc_create(int32_t num_blocks, int32_t block_size,
                                const int32_t* free_order, pkv_alloc_t** out) {
  if (!out) return fail(PKV_ERR_INVALID_ARG, "pkv_alloc_create: out is NULL");
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0)
    return fail(PKV_ERR_INVALID_ARG, "pkv_alloc_create: num_blocks=%d block_size=%d must be > 0",
                num_blocks, block_size);
  auto* a = new pkv_alloc;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->refcount.assign(num_blocks, 0);
  a->meta.assign(num_blocks, BlockMeta{});
  a->free_stack.resize(num_blocks);
  if (free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return fail(PKV_ERR_INVALID_ARG, "pkv_alloc_create: free_order is not a permutation (entry %d = %d)", i, b);
      }
      seen[b] = 1;
      a->free_stack[num_blocks - 1 - i] = b;
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) a->free_stack[num_blocks - 1 - i] = i;
  }
  *out = a;
  return pkv::ok();
}

extern "C" void pkv_alloc_destroy(pkv_alloc_t* a) { delete a; }

extern "C" int pkv_seq_add(pkv_alloc_t* a, int64_t seq_id, int32_t n_tokens) {
  if (!a) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_add: allocator is NULL");
  if (n_tokens < 0) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_add: n_tokens=%d < 0", n_tokens);
  if (a->seqs.count(seq_id)) return fail(PKV_ERR_SEQ_EXISTS, "pkv_seq_add: sequence %lld exists", (long long)seq_id);
  int64_t need = (static_cast<int64_t>(n_tokens) + a->block_size - 1) / a->block_size;
  if (need > a->available())
    return fail(PKV_ERR_OUT_OF_BLOCKS, "pkv_seq_add: needs %lld blocks, %lld free", (long long)need,
                (long long)a->available());
  Seq s;
  s.len = n_tokens;
  s.table.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.table.push_back(a->pop());
  a->seqs.emplace(seq_id, std::move(s));
  return pkv::ok();
}

extern "C" int pkv_seq_add_cached(pkv_alloc_t* a, int64_t seq_id, const int32_t* tokens, int32_t n_tokens,
                                  int32_t* n_cached_tokens) {
  if (!a || n_tokens < 0 || (n_tokens > 0 && !tokens))
    return fail(PKV_ERR_INVALID_ARG, "pkv_seq_add_cached: bad arguments");
  if (a->seqs.count(seq_id)) return fail(PKV_ERR_SEQ_EXISTS, "pkv_seq_add_cached: sequence %lld exists", (long long)seq_id);
  const int32_t bs = a->block_size;
  if (a->block_tokens.empty()) {  // first use of the prefix cache
    a->block_tokens.assign(static_cast<size_t>(a->num_blocks) * bs, 0);
    a->cache.reserve(static_cast<size_t>(a->num_blocks));
  }
  const int32_t nfull = n_tokens / bs;
  const int32_t nblk = (n_tokens + bs - 1) / bs;
  // chain hashes of the full blocks; the leading run found in the cache
  std::vector<uint64_t> h(nfull);
  uint64_t prev = kFnvBasis;
  for (int32_t i = 0; i < nfull; ++i) {
    h[i] = fnv1a(prev, tokens + static_cast<int64_t>(i) * bs, static_cast<size_t>(bs));
    prev = h[i];
  }
  std::vector<int32_t> hit_blocks;
  int64_t revived = 0;
  for (int32_t i = 0; i < nfull; ++i) {
    const int32_t b = a->lookup(h[i], i ? h[i - 1] : kFnvBasis, tokens + static_cast<int64_t>(i) * bs);
    if (b < 0) break;
    hit_blocks.push_back(b);
    if (a->refcount[b] == 0) ++revived;
  }
  const int32_t hits = static_cast<int32_t>(hit_blocks.size());
  const int64_t need = nblk - hits;
  if (need > a->available() - revived)
    return fail(PKV_ERR_OUT_OF_BLOCKS, "pkv_seq_add_cached: needs %lld new blocks, %lld available",
                (long long)need, (long long)(a->available() - revived));
  a->cache_queries += nfull;
  a->cache_hits += hits;
  Seq s;
  s.len = n_tokens;
  s.table.reserve(nblk);
  for (int32_t b : hit_blocks) {
    if (a->refcount[b] == 0) a->lru_remove(b);
    a->refcount[b] += 1;
    s.table.push_back(b);
  }
  for (int32_t i = hits; i < nblk; ++i) {
    const int32_t b = a->pop();
    s.table.push_back(b);
    if (i < nfull && a->cache.find(h[i]) == a->cache.end()) {  // register the new full block
      BlockMeta& m = a->meta[b];
      m.registered = true;
      m.key = h[i];
      m.parent = i ? h[i - 1] : kFnvBasis;
      std::copy(tokens + static_cast<int64_t>(i) * bs, tokens + static_cast<int64_t>(i + 1) * bs,
                a->block_tokens.begin() + static_cast<int64_t>(b) * bs);
      a->cache.emplace(h[i], b);
    }
  }
  a->seqs.emplace(seq_id, std::move(s));
  if (n_cached_tokens) *n_cached_tokens = hits * bs;
  return pkv::ok();
}

extern "C" int pkv_seq_fork(pkv_alloc_t* a, int64_t parent, int64_t child) {
  if (!a) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_fork: allocator is NULL");
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end()) return fail(PKV_ERR_UNKNOWN_SEQ, "pkv_seq_fork: unknown parent %lld", (long long)parent);
  if (a->seqs.count(child)) return fail(PKV_ERR_SEQ_EXISTS, "pkv_seq_fork: child %lld exists", (long long)child);
  Seq s = it->second;  // copy before emplace may rehash
  for (int32_t b : s.table) a->refcount[b] += 1;
  a->seqs.emplace(child, std::move(s));
  return pkv::ok();
}

extern "C" int pkv_seq_append_slots(pkv_alloc_t* a, const int64_t* seq_ids, int32_t n,
                                    int32_t* slot_out, int32_t* cow_pairs_out, int32_t cow_capacity,
                                    int32_t* n_cow) {
  if (!a) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_append_slots: allocator is NULL");
  if (n < 0 || (n > 0 && (!seq_ids || !slot_out)) || !n_cow || (cow_capacity > 0 && !cow_pairs_out))
    return fail(PKV_ERR_INVALID_ARG, "pkv_seq_append_slots: bad arguments");
  const int32_t bs = a->block_size;
  auto& undo = a->undo;
  undo.clear();
  int32_t ncow = 0;
  int rc = PKV_OK;
  for (int32_t i = 0; i < n && rc == PKV_OK; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) {
      rc = fail(PKV_ERR_UNKNOWN_SEQ, "pkv_seq_append_slots: unknown sequence %lld", (long long)seq_ids[i]);
      break;
    }
    Seq& s = it->second;
    const int32_t pos = s.len;
    const int32_t bi = pos / bs, off = pos % bs;
    if (off == 0) {
      if (a->available() == 0) {
        rc = fail(PKV_ERR_OUT_OF_BLOCKS, "pkv_seq_append_slots: no free block for sequence %lld",
                  (long long)seq_ids[i]);
        break;
      }
      bool evicted = false;
      int32_t b = a->pop(&evicted);
      undo.push_back({evicted ? Undo::kPopEvicted : Undo::kPop, nullptr, b, 0});
      s.table.push_back(b);
      undo.push_back({Undo::kTablePush, &s, 0, 0});
    } else {
      const int32_t old = s.table[bi];
      if (a->refcount[old] > 1) {
        if (a->available() == 0) {
          rc = fail(PKV_ERR_OUT_OF_BLOCKS, "pkv_seq_append_slots: no free block to copy shared block %d", old);
          break;
        }
        if (ncow >= cow_capacity) {
          rc = fail(PKV_ERR_INVALID_ARG, "pkv_seq_append_slots: cow_capacity %d too small", cow_capacity);
          break;
        }
        bool evicted = false;
        int32_t fresh = a->pop(&evicted);
        undo.push_back({evicted ? Undo::kPopEvicted : Undo::kPop, nullptr, fresh, 0});
        a->refcount[old] -= 1;
        undo.push_back({Undo::kRefDec, nullptr, old, 0});
        s.table[bi] = fresh;
        undo.push_back({Undo::kTableSet, &s, bi, old});
        cow_pairs_out[2 * ncow] = old;
        cow_pairs_out[2 * ncow + 1] = fresh;
        ++ncow;
        a->cow_copies += 1;
        undo.push_back({Undo::kCow, nullptr, 0, 0});
      }
    }
    slot_out[i] = s.table[bi] * bs + off;
    undo.push_back({Undo::kLen, &s, pos, 0});
    s.len = pos + 1;
  }
  if (rc != PKV_OK) {
    for (auto u = undo.rbegin(); u != undo.rend(); ++u) {
      switch (u->kind) {
        case Undo::kPop: a->refcount[u->a] = 0; a->free_stack.push_back(u->a); break;
        case Undo::kPopEvicted: {  // re-register the evicted block at the front of the cached-free list
          BlockMeta& m = a->meta[u->a];
          a->refcount[u->a] = 0;
          m.registered = true;
          a->cache.emplace(m.key, u->a);
          a->lru_push_front(u->a);
          break;
        }
        case Undo::kTablePush: u->seq->table.pop_back(); break;
        case Undo::kTableSet: u->seq->table[u->a] = u->b; break;
        case Undo::kRefDec: a->refcount[u->a] += 1; break;
        case Undo::kLen: u->seq->len = u->a; break;
        case Undo::kCow: a->cow_copies -= 1; break;
      }
    }
    *n_cow = 0;
    return rc;
  }
  *n_cow = ncow;
  return pkv::ok();
}

extern "C" int pkv_seq_free(pkv_alloc_t* a, int64_t seq_id) {
  if (!a) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_free: allocator is NULL");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(PKV_ERR_UNKNOWN_SEQ, "pkv_seq_free: unknown sequence %lld", (long long)seq_id);
  for (int32_t b : it->second.table) {
    if (--a->refcount[b] == 0) a->release(b);
  }
  a->seqs.erase(it);
  return pkv::ok();
}

extern "C" int pkv_seq_len(const pkv_alloc_t* a, int64_t seq_id, int32_t* len) {
  if (!a || !len) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_len: NULL argument");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(PKV_ERR_UNKNOWN_SEQ, "pkv_seq_len: unknown sequence %lld", (long long)seq_id);
  *len = it->second.len;
  return pkv::ok();
}

extern "C" int pkv_block_tables(const pkv_alloc_t* a, const int64_t* seq_ids, int32_t n, int32_t max_blocks,
                                int32_t* tables_out, int32_t* seq_lens_out) {
  if (!a || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || (max_blocks > 0 && !tables_out))))
    return fail(PKV_ERR_INVALID_ARG, "pkv_block_tables: bad arguments");
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) return fail(PKV_ERR_UNKNOWN_SEQ, "pkv_block_tables: unknown sequence %lld", (long long)seq_ids[i]);
    if (static_cast<int32_t>(it->second.table.size()) > max_blocks)
      return fail(PKV_ERR_INVALID_ARG, "pkv_block_tables: sequence %lld has %zu blocks > max_blocks %d",
                  (long long)seq_ids[i], it->second.table.size(), max_blocks);
  }
  for (int32_t i = 0; i < n; ++i) {
    const Seq& s = a->seqs.find(seq_ids[i])->second;
    int32_t* row = tables_out + static_cast<int64_t>(i) * max_blocks;
    std::copy(s.table.begin(), s.table.end(), row);
    std::fill(row + s.table.size(), row + max_blocks, -1);
    if (seq_lens_out) seq_lens_out[i] = s.len;
  }
  return pkv::ok();
}

extern "C" int pkv_alloc_stats(const pkv_alloc_t* a, pkv_stats_t* out) {
  if (!a || !out) return fail(PKV_ERR_INVALID_ARG, "pkv_alloc_stats: NULL argument");
  const int32_t bs = a->block_size;
  std::vector<int32_t> fill(a->num_blocks, 0);
  int64_t logical = 0;
  for (const auto& kv : a->seqs) {
    const Seq& s = kv.second;
    logical += s.len;
    for (size_t i = 0; i < s.table.size(); ++i) {
      int32_t used = std::min<int64_t>(bs, s.len - static_cast<int64_t>(i) * bs);
      int32_t& f = fill[s.table[i]];
      f = std::max(f, used);
    }
  }
  int64_t waste = 0;
  for (int32_t b = 0; b < a->num_blocks; ++b)
    if (a->refcount[b] > 0) waste += bs - fill[b];
  out->num_blocks = a->num_blocks;
  out->block_size = bs;
  out->free_blocks = a->available();
  out->used_blocks = a->num_blocks - out->free_blocks;
  out->num_seqs = static_cast<int64_t>(a->seqs.size());
  out->cow_copies = a->cow_copies;
  out->logical_tokens = logical;
  out->waste_tokens = waste;
  out->cached_blocks = static_cast<int64_t>(a->cache.size());
  out->cache_queries = a->cache_queries;
  out->cache_hits = a->cache_hits;
  return pkv::ok();
}
