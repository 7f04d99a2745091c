// Host-side block allocator: free stack, per-block reference counts,
// copy-on-write on a write into a shared block, all-or-nothing errors.
//
// Follows "vLLM's 'memory paging' — PagedAttention illustrated":
//   §2        fixed-size pages, a page table per sequence, a free page list;
//   §3 ph. 1  the token after a full page takes a new page, the table grows;
//   §3 ph. 3  shared prefix pages carry a reference count and are reclaimed
//             by the last sharer ("copy-on-write" style sharing);
//   §4        admission refuses requests that do not fit; abort frees pages.
// Every operation is O(1) per token (O(blocks) for free/fork/tables); none
// touches the GPU.
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
  enum Kind { kPop, kTablePush, kTableSet, kRefDec, kLen, kCow } kind;
  Seq* seq;
  int32_t a;  // block id, table index or old length
  int32_t b;  // old table value
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

  int32_t pop() {
    int32_t b = free_stack.back();
    free_stack.pop_back();
    refcount[b] = 1;
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
  if (need > static_cast<int64_t>(a->free_stack.size()))
    return fail(PKV_ERR_OUT_OF_BLOCKS, "pkv_seq_add: needs %lld blocks, %zu free", (long long)need,
                a->free_stack.size());
  Seq s;
  s.len = n_tokens;
  s.table.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.table.push_back(a->pop());
  a->seqs.emplace(seq_id, std::move(s));
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
      if (a->free_stack.empty()) {
        rc = fail(PKV_ERR_OUT_OF_BLOCKS, "pkv_seq_append_slots: no free block for sequence %lld",
                  (long long)seq_ids[i]);
        break;
      }
      int32_t b = a->pop();
      undo.push_back({Undo::kPop, nullptr, b, 0});
      s.table.push_back(b);
      undo.push_back({Undo::kTablePush, &s, 0, 0});
    } else {
      const int32_t old = s.table[bi];
      if (a->refcount[old] > 1) {
        if (a->free_stack.empty()) {
          rc = fail(PKV_ERR_OUT_OF_BLOCKS, "pkv_seq_append_slots: no free block to copy shared block %d", old);
          break;
        }
        if (ncow >= cow_capacity) {
          rc = fail(PKV_ERR_INVALID_ARG, "pkv_seq_append_slots: cow_capacity %d too small", cow_capacity);
          break;
        }
        int32_t fresh = a->pop();
        undo.push_back({Undo::kPop, nullptr, fresh, 0});
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
    if (--a->refcount[b] == 0) a->free_stack.push_back(b);
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
  out->free_blocks = static_cast<int64_t>(a->free_stack.size());
  out->used_blocks = a->num_blocks - out->free_blocks;
  out->num_seqs = static_cast<int64_t>(a->seqs.size());
  out->cow_copies = a->cow_copies;
  out->logical_tokens = logical;
  out->waste_tokens = waste;
  return pkv::ok();
}
