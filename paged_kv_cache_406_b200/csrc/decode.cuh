// PagedAttention decode for sm_100a.
//
// What is computed ("vLLM's 'memory paging' — PagedAttention illustrated",
// §3 phase 2): for every sequence b and query head h the kernel follows b's
// block table, treats the scattered physical blocks as one logically
// contiguous K and V, and returns softmax(scale · q·Kᵀ)·V, with query head h
// reading KV head h / G (grouped-query attention, contiguous groups).
//
// How (B200 design, not the page's):
//   plan kernel    one CTA turns seq_lens into a work list of partitions of
//                  `partition_tokens` tokens, largest first (in a decode step
//                  the launch that builds it also writes the step's new K/V
//                  rows: append_plan_kernel);
//   decode kernel  persistent CTAs (grid = SMs x resident CTAs) walk the list
//                  in rounds of alternating direction (unit_index); per work
//                  unit (sequence, partition, KV
//                  head) a producer warp streams each block's K and V tiles
//                  (one contiguous block_size x head_dim tile each) into a
//                  shared-memory ring with 1-D bulk copies completing on
//                  mbarriers; four consumer warps take every fourth block and
//                  keep their own online softmax state (running max m, sum l,
//                  fp32 accumulator), and merge at the end of the unit;
//   merge kernel   for sequences that were split, one warp per (sequence,
//                  query head) merges the per-partition (m, l, o) with the
//                  max/sum rescaling
//                      out = Σ_p 2^(m_p-M) o_p / Σ_p 2^(m_p-M) l_p.
// Scores are kept in log2 units (q is pre-multiplied by scale·log2 e).  The
// running max is only moved when a new score exceeds it by more than
// kRescaleThreshold (2^8 headroom in fp32), which leaves the result unchanged
// because every accumulator and sum is always taken against the same m.
#pragma once

#include "device_common.cuh"

namespace pkv {

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr float kRescaleThreshold = 8.0f;
constexpr unsigned kFull = 0xffffffffu;

// A batch may span up to kMaxPools pools of different block sizes (one pool
// per block-size class): sequences seq0 .. of pool c (up to the next pool's
// seq0) are rows (b - seq0) of that pool's block table.
constexpr int kMaxPools = 3;

struct PoolView {
  const void* k;          // K and V pools [num_blocks][num_kv_heads][block_size][head_dim]
  const void* v;
  const int32_t* tables;  // [sequences of the pool][max_blocks]
  int32_t num_blocks, max_blocks, block_size, seq0;
};

struct DecodeParams {
  const void* q;
  PoolView pool[kMaxPools];
  int32_t n_pools;
  int32_t num_q_heads, num_kv_heads, partition_tokens, max_parts;
  int32_t n_stages;
  float scale_log2;
  float v_scale;  // multiplies the output (e4m3 V pools; 1 otherwise)
  const int4* items;  // {b, partition, partitions of b, end token}
  const int32_t* n_items;
  float* part_m;
  float* part_l;
  float* part_o;
  float* out;
  // Test support for the bounded waits (pkv_debug_stall_decode): the
  // producer of CTA `stall_cta` skips the copies of that CTA's first work
  // unit, so its consumers' waits run out.  stall_cta < 0 in normal calls.
  int32_t stall_cta;
};

// Pool of sequence b (0 for single-pool batches).
__device__ __forceinline__ int pool_of(const PoolView* pool, int n_pools, int b) {
  return n_pools == 1 ? 0 : (b >= pool[1].seq0 ? 1 : 0) + (n_pools > 2 && b >= pool[2].seq0 ? 1 : 0);
}

// Element c of a small array held in kernel parameters, by selects (a
// dynamic index into the parameter space would copy the array to local
// memory).
template <typename V>
__device__ __forceinline__ V pick3(const V (&a)[kMaxPools], int c) {
  return c == 0 ? a[0] : (c == 1 ? a[1] : a[2]);
}

// ---------------------------------------------------------------------------
// plan: seq_lens -> work list, partitions sorted by size, largest first
// ---------------------------------------------------------------------------
struct PlanArgs {
  const int32_t* seq_lens;
  int32_t num_seqs, part_tokens;
  int32_t bin_tokens;  // size classes of the sort: part_tokens / bin_tokens + 1 bins
  int32_t n_pools;
  int32_t seq0[kMaxPools];  // first sequence of each pool
  int32_t cap[kMaxPools];   // tokens a sequence of the pool can hold (max_blocks * block_size)
};

// One CTA builds the list; `hist` is 2 * (part_tokens / bin_tokens + 1) ints
// of shared memory.  A length outside [0, its pool's capacity] is recorded
// and clamped.
__device__ __forceinline__ int plan_len(const PlanArgs& a, int b, bool record) {
  int c = 0;
  if (a.n_pools > 1) c = (b >= a.seq0[1] ? 1 : 0) + (a.n_pools > 2 && b >= a.seq0[2] ? 1 : 0);
  const int cap = pick3(a.cap, c);
  int L = a.seq_lens[b];
  if (L < 0 || L > cap) {
    if (record) record_error(PKV_ERR_BAD_BLOCK);
    L = L < 0 ? 0 : cap;
  }
  return L;
}

__device__ __forceinline__ void plan_body(const PlanArgs& a, int4* __restrict__ items, int32_t* __restrict__ n_items,
                                          int32_t* hist) {
  const int part_tokens = a.part_tokens, bin = a.bin_tokens;
  const int kmax = part_tokens / bin;
  int32_t* cursor = hist + kmax + 1;
  for (int i = threadIdx.x; i <= kmax; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int b = threadIdx.x; b < a.num_seqs; b += blockDim.x) {
    const int L = plan_len(a, b, true);
    const int nfull = L / part_tokens, rem = L % part_tokens;
    if (nfull) atomicAdd(&hist[kmax], nfull);
    if (rem) atomicAdd(&hist[(rem + bin - 1) / bin], 1);
    if (L == 0) atomicAdd(&hist[0], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int k = kmax; k >= 0; --k) {
      cursor[k] = run;
      run += hist[k];
    }
    *n_items = run;
  }
  __syncthreads();
  for (int b = threadIdx.x; b < a.num_seqs; b += blockDim.x) {
    const int L = plan_len(a, b, false);
    const int nfull = L / part_tokens, rem = L % part_tokens;
    if (nfull) {
      int pos = atomicAdd(&cursor[kmax], nfull);
      for (int p = 0; p < nfull; ++p)
        items[pos + p] = make_int4(b, p, nfull + (rem ? 1 : 0), (p + 1) * part_tokens);
    }
    if (rem) {
      int pos = atomicAdd(&cursor[(rem + bin - 1) / bin], 1);
      items[pos] = make_int4(b, nfull, nfull + 1, L);
    }
    if (L == 0) {
      int pos = atomicAdd(&cursor[0], 1);
      items[pos] = make_int4(b, 0, 1, 0);
    }
  }
}

__global__ void __launch_bounds__(1024) plan_kernel(const PlanArgs a, int4* __restrict__ items,
                                                    int32_t* __restrict__ n_items) {
  // launched programmatically serialised: the previous kernel of the stream
  // (which may have produced the lengths) is complete before anything is read
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the decode grid may be scheduled now; it waits for this grid's results
  // (griddepcontrol.wait) before reading them
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ int32_t hist[];  // [kmax + 1] counts, then [kmax + 1] cursors
  plan_body(a, items, n_items, hist);
}

// ---------------------------------------------------------------------------
// cross-lane helpers within a group of 8 lanes that share one token row
// ---------------------------------------------------------------------------

// Sums G per-lane partial dot products over the 8 lanes of a token group and
// leaves each lane with the full score of one head, head_of<G>(r8).
template <int G>
__device__ __forceinline__ float reduce_scatter(const float (&v)[G], int r8) {
  if constexpr (G == 1) {
    float x = v[0];
    x += __shfl_xor_sync(kFull, x, 4);
    x += __shfl_xor_sync(kFull, x, 2);
    x += __shfl_xor_sync(kFull, x, 1);
    return x;
  } else if constexpr (G == 2) {
    const bool u4 = r8 & 4;
    float x = (u4 ? v[1] : v[0]) + __shfl_xor_sync(kFull, u4 ? v[0] : v[1], 4);
    x += __shfl_xor_sync(kFull, x, 2);
    x += __shfl_xor_sync(kFull, x, 1);
    return x;
  } else {
    static_assert(G == 4, "group size");
    const bool u4 = r8 & 4, u2 = r8 & 2;
    float a0 = (u4 ? v[2] : v[0]) + __shfl_xor_sync(kFull, u4 ? v[0] : v[2], 4);
    float a1 = (u4 ? v[3] : v[1]) + __shfl_xor_sync(kFull, u4 ? v[1] : v[3], 4);
    float x = (u2 ? a1 : a0) + __shfl_xor_sync(kFull, u2 ? a0 : a1, 2);
    x += __shfl_xor_sync(kFull, x, 1);
    return x;
  }
}

template <int G>
__device__ __forceinline__ int head_of(int r8) {
  if constexpr (G == 1) return 0;
  else if constexpr (G == 2) return (r8 >> 2) & 1;
  else return ((r8 >> 2) & 1) * 2 + ((r8 >> 1) & 1);
}

// The lane of each head that writes per-head values (one per duplicate set).
template <int G>
__device__ __forceinline__ bool head_writer(int r8) {
  if constexpr (G == 1) return r8 == 0;
  else if constexpr (G == 2) return (r8 & 3) == 0;
  else return (r8 & 1) == 0;
}

// Inverse of reduce_scatter's layout: every lane of the token group ends with
// all G values, out[h] = value held by the lanes of head h.
template <int G>
__device__ __forceinline__ void all_gather(float x, float (&out)[G], int r8) {
  if constexpr (G == 1) {
    out[0] = x;
  } else if constexpr (G == 2) {
    const bool u4 = r8 & 4;
    float y = __shfl_xor_sync(kFull, x, 4);
    out[0] = u4 ? y : x;
    out[1] = u4 ? x : y;
  } else {
    const bool u4 = r8 & 4, u2 = r8 & 2;
    float y = __shfl_xor_sync(kFull, x, 2);
    float lo = u2 ? y : x, hi = u2 ? x : y;
    float y0 = __shfl_xor_sync(kFull, lo, 4);
    float y1 = __shfl_xor_sync(kFull, hi, 4);
    out[0] = u4 ? y0 : lo;
    out[1] = u4 ? y1 : hi;
    out[2] = u4 ? lo : y0;
    out[3] = u4 ? hi : y1;
  }
}

// v[head_of<G>(r8)] without dynamic register indexing.
template <int G>
__device__ __forceinline__ float pick(const float (&v)[G], int r8) {
  if constexpr (G == 1) return v[0];
  else if constexpr (G == 2) return (r8 & 4) ? v[1] : v[0];
  else {
    const bool u4 = r8 & 4, u2 = r8 & 2;
    return u4 ? (u2 ? v[3] : v[2]) : (u2 ? v[1] : v[0]);
  }
}

struct WorkUnit {
  int b, part, nparts, t0, t1, g, nblk, c;  // c: the pool of sequence b
};

// The work unit this CTA takes in round r of the persistent loop.  Rounds go
// forward and backward in turn over the largest-first list: the CTA that
// takes a round's largest unit takes the next round's smallest, so the
// per-CTA sums even out (on the Llama-3-8B-shaped batch the most loaded CTA
// has 1 % more tokens than the mean instead of 6 % with a plain stride).
__device__ __forceinline__ int unit_index(int r) {
  const int c = (r & 1) ? static_cast<int>(gridDim.x - 1 - blockIdx.x) : static_cast<int>(blockIdx.x);
  return r * static_cast<int>(gridDim.x) + c;
}

// kMulti: the batch may span several pools (else pool 0 only, known at
// compile time).
template <bool kMulti = false>
__device__ __forceinline__ WorkUnit load_unit(const DecodeParams& p, int w) {
  WorkUnit u;
  const int idx = w / p.num_kv_heads;
  u.g = w - idx * p.num_kv_heads;
  const int4 it = p.items[idx];
  u.b = it.x;
  u.part = it.y;
  u.nparts = it.z;
  u.t0 = it.y * p.partition_tokens;
  u.t1 = it.w;
  u.c = kMulti ? pool_of(p.pool, p.n_pools, u.b) : 0;
  const int bs = kMulti ? pick3(p.pool, u.c).block_size : p.pool[0].block_size;
  u.nblk = (u.t1 - u.t0 + bs - 1) / bs;
  return u;
}

// Final merge of one work unit: the kCW per-warp records in `rec`
// (acc[G][D], m[G], l[G] each, taken against each warp's own running max)
// are rescaled to their common max and either normalised into `out` (the
// sequence has one partition) or stored as the partition's (m, l, o) partial
// for merge_kernel.  Called by the consumer threads (0 .. kCW*32-1)
// after the named barrier that publishes the records.
template <int G, int D, int kCW = kConsumerWarps>
__device__ __forceinline__ void merge_store(const float* rec, const WorkUnit& u, const DecodeParams& p) {
  constexpr int kMF = G * D + 2 * G;
  const bool single = u.nparts == 1;
  for (int idx = threadIdx.x; idx < G * D; idx += kCW * 32) {
    const int h = idx / D, d = idx - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < kCW; ++w2) M = fmaxf(M, rec[w2 * kMF + G * D + h]);
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w2 = 0; w2 < kCW; ++w2) {
        const float f = fast_exp2(rec[w2 * kMF + G * D + h] - M);
        num += f * rec[w2 * kMF + h * D + d];
        den += f * rec[w2 * kMF + G * D + G + h];
      }
    }
    const int64_t row = static_cast<int64_t>(u.b) * p.num_q_heads + u.g * G + h;
    if (single) {
      p.out[row * D + d] = den > 0.f ? p.v_scale * num / den : 0.f;
    } else {
      const int64_t pr = row * p.max_parts + u.part;
      p.part_o[pr * D + d] = p.v_scale * num;
      if (d == 0) {
        p.part_m[pr] = M;
        p.part_l[pr] = den;
      }
    }
  }
}

// Shared memory: [n_stages][K tile | V tile] ring, 2 x kConsumerWarps merge
// records, full/empty mbarriers, abort flag.
template <typename T, int D, int G>
struct DecodeSmem {
  static constexpr int kMergeFloats = G * D + 2 * G;  // acc[G][D], m[G], l[G]
  __host__ __device__ static size_t ring_bytes(int bs, int ns) { return size_t(ns) * 2 * bs * D * sizeof(T); }
  __host__ __device__ static size_t bytes(int bs, int ns) {
    // + 16: abort and merge flags; + 128: the producer's window of 32 block-table entries
    return ring_bytes(bs, ns) + 2 * kConsumerWarps * kMergeFloats * sizeof(float) + 2 * ns * sizeof(uint64_t) + 16 +
           128;
  }
};

// kStall: the instance that honours DecodeParams::stall_cta (the test of the
// bounded waits); production launches use the instance without the check.
template <typename T, int D, int G, bool kStall = false>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kVec = Elem<T>::kVec;       // elements per 16-byte chunk
  constexpr int kChunksPerLane = D / kVec / 8;  // 8 lanes cover one token row
  constexpr int kPairs = kChunksPerLane * kVec / 2;  // fp32 pairs per lane
  constexpr int kMF = DecodeSmem<T, D, G>::kMergeFloats;
  static_assert(kChunksPerLane >= 1, "head_dim too small");

  const int BS = p.pool[0].block_size;  // one pool: the multi-pool batches take the tensor-core kernel
  const int NS = p.n_stages;
  const uint32_t tile_bytes = BS * D * sizeof(T);
  const uint32_t stage_bytes = 2 * tile_bytes;
  float* merge = reinterpret_cast<float*>(smem + DecodeSmem<T, D, G>::ring_bytes(BS, NS));
  uint64_t* full = reinterpret_cast<uint64_t*>(merge + 2 * kConsumerWarps * kMF);
  uint64_t* empty = full + NS;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NS);
  int32_t* tab = reinterpret_cast<int32_t*>(empty + NS) + 4;  // 32 block-table entries
  const uint32_t ring_s = smem_addr(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_addr(full + s), 1);
      mbar_init(smem_addr(empty + s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the plan kernel's work list is complete
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // let merge_kernel be scheduled

  const int n_work = *p.n_items * p.num_kv_heads;
  const int Hq = p.num_q_heads;

  if (warp == kConsumerWarps) {
    // ----------------------------- producer -----------------------------
    // All lanes walk the units and refill a 32-entry block-table window in
    // shared memory; lane 0 alone issues the window's blocks (no warp-wide
    // synchronisation on the per-block path).
    const uint64_t policy = l2_evict_first_policy();
    const uint64_t tab_policy = l2_evict_last_policy();
    const unsigned char* kbase = static_cast<const unsigned char*>(p.pool[0].k);
    const unsigned char* vbase = static_cast<const unsigned char*>(p.pool[0].v);
    int s = 0;
    uint32_t ph = 0, issued = 0, skipped = 0;  // stage uses so far; the first `skipped` of them issued no copy
    bool ok = true;
    for (int r = 0, w = unit_index(0); w < n_work && ok; w = unit_index(++r)) {
      const bool stall = kStall && r == 0 && p.stall_cta == static_cast<int>(blockIdx.x);
      const WorkUnit u = load_unit(p, w);
      const int32_t* trow = p.pool[0].tables + static_cast<int64_t>(u.b) * p.pool[0].max_blocks + u.t0 / BS;
      for (int jb = 0; jb < u.nblk && ok; jb += 32) {
        tab[lane] = jb + lane < u.nblk ? ld_table(trow + jb + lane, tab_policy) : 0;
        __syncwarp();
        if (lane == 0) {
          const int cnt = min(32, u.nblk - jb);
          for (int j = 0; j < cnt; ++j) {
            if (!mbar_wait(smem_addr(empty + s), ph ^ 1, abort_flag)) {
              record_error(PKV_ERR_DEVICE_TIMEOUT);
              *abort_flag = 1;
              ok = false;
              break;
            }
            int phys = tab[j];
            if (static_cast<unsigned>(phys) >= static_cast<unsigned>(p.pool[0].num_blocks)) {
              record_error(PKV_ERR_BAD_BLOCK);
              phys = 0;
            }
            const size_t off = (static_cast<size_t>(phys) * p.num_kv_heads + u.g) * tile_bytes;
            const uint32_t bar = smem_addr(full + s);
            if (!stall) {
              mbar_arrive_expect_tx(bar, stage_bytes);
              bulk_g2s(ring_s + s * stage_bytes, kbase + off, tile_bytes, bar, policy);
              bulk_g2s(ring_s + s * stage_bytes + tile_bytes, vbase + off, tile_bytes, bar, policy);
            } else {
              ++skipped;  // nothing will land in this stage: its consumer's wait runs out
            }
            ++issued;
            if (++s == NS) {
              s = 0;
              ph ^= 1;
            }
          }
        }
        __syncwarp();
        ok = __shfl_sync(kFull, ok, 0);
      }
    }
    // Before the CTA exits no copy may still be landing in its shared memory:
    // wait (bounded) for the last phase issued into every stage whose last use
    // carried a copy.
    if (lane == 0) {
      for (int st = 0; st < NS && st < static_cast<int>(issued); ++st) {
        const uint32_t uses = (issued - st + NS - 1) / NS;
        if (st + NS * (uses - 1) < skipped) continue;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(smem_addr(full + st), (uses - 1) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    return;
  }

  // ------------------------------ consumers ------------------------------
  const int r8 = lane & 7, tg = lane >> 3;
  const int hs = head_of<G>(r8);
  const bool writer = head_writer<G>(r8);
  uint32_t c = 0;
  int iter = 0;
  bool ok = true;
  for (int w = unit_index(0); w < n_work; w = unit_index(++iter)) {
    const WorkUnit u = load_unit(p, w);

    // q rows of this KV head's G query heads, my dims, scaled to log2 units
    float2 q2[G][kPairs];
    {
      const T* qrow = static_cast<const T*>(p.q) + (static_cast<int64_t>(u.b) * Hq + u.g * G) * D;
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int i = 0; i < kChunksPerLane; ++i) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow + h * D + (r8 + 8 * i) * kVec));
          float2 f[kVec / 2];
          Elem<T>::widen(raw, f);
#pragma unroll
          for (int e = 0; e < kVec / 2; ++e)
            q2[h][i * kVec / 2 + e] = make_float2(f[e].x * p.scale_log2, f[e].y * p.scale_log2);
        }
      }
    }

    float m[G];
    float2 acc[G][kPairs];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
#pragma unroll
      for (int e = 0; e < kPairs; ++e) acc[h][e] = make_float2(0.f, 0.f);
    }
    float m_own = -INFINITY, l_own = 0.f;

    const int j0 = (warp - static_cast<int>(c % kConsumerWarps) + kConsumerWarps) % kConsumerWarps;
    int s = (c + j0) % NS;
    uint32_t ph = ((c + j0) / NS) & 1;
    for (int j = j0; j < u.nblk && ok; j += kConsumerWarps) {
      const bool landed = __all_sync(kFull, mbar_wait(smem_addr(full + s), ph, abort_flag));
      if (!landed) {
        if (lane == 0) {
          record_error(PKV_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
        }
        ok = false;
        break;
      }
      const unsigned char* ks = smem + s * stage_bytes;
      const unsigned char* vs = ks + tile_bytes;
      const int nv = min(BS, u.t1 - (u.t0 + j * BS));
      const int nrows = (nv + 3) >> 2;
      for (int rr = 0; rr < nrows; ++rr) {
        const int tt = rr * 4 + tg;
        const bool valid = tt < nv;
        const unsigned char* krow = ks + tt * (D * sizeof(T));
        float part[G];
        {
          float2 pp[G];
#pragma unroll
          for (int h = 0; h < G; ++h) pp[h] = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < kChunksPerLane; ++i) {
            const uint4 raw = *reinterpret_cast<const uint4*>(krow + (r8 + 8 * i) * 16);
            float2 kf[kVec / 2];
            Elem<T>::widen(raw, kf);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int e = 0; e < kVec / 2; ++e) pp[h] = __ffma2_rn(q2[h][i * kVec / 2 + e], kf[e], pp[h]);
          }
#pragma unroll
          for (int h = 0; h < G; ++h) part[h] = pp[h].x + pp[h].y;
        }
        float s_own = reduce_scatter<G>(part, r8);
        s_own = valid ? s_own : -INFINITY;

        if (__any_sync(kFull, s_own > m_own + kRescaleThreshold)) {
          float mx = s_own;
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
          float mall[G], fac[G];
          all_gather<G>(mx, mall, r8);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float mn = fmaxf(m[h], mall[h]);
            fac[h] = (mn == -INFINITY) ? 1.f : fast_exp2(m[h] - mn);
            m[h] = mn;
#pragma unroll
            for (int e = 0; e < kPairs; ++e) acc[h][e] = __fmul2_rn(acc[h][e], make_float2(fac[h], fac[h]));
          }
          l_own *= pick<G>(fac, r8);
          m_own = pick<G>(m, r8);
        }
        const float p_own = fast_exp2(s_own - m_own);
        l_own += p_own;
        float pv[G];
        all_gather<G>(p_own, pv, r8);
        if (valid) {
          const unsigned char* vrow = vs + tt * (D * sizeof(T));
#pragma unroll
          for (int i = 0; i < kChunksPerLane; ++i) {
            const uint4 raw = *reinterpret_cast<const uint4*>(vrow + (r8 + 8 * i) * 16);
            float2 vf[kVec / 2];
            Elem<T>::widen(raw, vf);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int e = 0; e < kVec / 2; ++e)
                acc[h][i * kVec / 2 + e] = __ffma2_rn(make_float2(pv[h], pv[h]), vf[e], acc[h][i * kVec / 2 + e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(empty + s));
      s += kConsumerWarps;
      if (s >= NS) {
        s -= NS;
        ph ^= 1;
      }
    }
    c += u.nblk;

    // ---- merge the 4 token groups of this warp, then the 4 warps ----
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < kPairs; ++e) {
        acc[h][e].x += __shfl_xor_sync(kFull, acc[h][e].x, 8);
        acc[h][e].y += __shfl_xor_sync(kFull, acc[h][e].y, 8);
        acc[h][e].x += __shfl_xor_sync(kFull, acc[h][e].x, 16);
        acc[h][e].y += __shfl_xor_sync(kFull, acc[h][e].y, 16);
      }
    l_own += __shfl_xor_sync(kFull, l_own, 8);
    l_own += __shfl_xor_sync(kFull, l_own, 16);

    float* mb = merge + ((iter & 1) * kConsumerWarps + warp) * kMF;
    if (tg == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < kChunksPerLane; ++i)
#pragma unroll
          for (int e = 0; e < kVec / 2; ++e)
            *reinterpret_cast<float2*>(mb + h * D + (r8 + 8 * i) * kVec + 2 * e) = acc[h][i * kVec / 2 + e];
      if (writer) mb[G * D + G + hs] = l_own;
    }
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) mb[G * D + h] = m[h];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");

    merge_store<G, D>(merge + (iter & 1) * kConsumerWarps * kMF, u, p);
  }
}

// ---------------------------------------------------------------------------
// merge: partitions of split sequences; one warp per (sequence, query head).
// Lanes first hold the rescale weight 2^(m_p - M) and l_p of 32 partitions
// each; the weighted rows o_p are then summed with several partitions' loads
// in flight.  The length, the first 32 (m, l) pairs and the first 4 rows are
// loaded in one round, before the partition count they depend on is known.
// Launched with programmatic serialisation after the decode kernel: it waits
// (griddepcontrol.wait) for all partials before reading.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const int32_t* __restrict__ seq_lens, int32_t num_seqs,
                                                    int32_t num_q_heads, int32_t max_tokens, int32_t part_tokens,
                                                    int32_t max_parts, const float* __restrict__ part_m,
                                                    const float* __restrict__ part_l,
                                                    const float* __restrict__ part_o, float* __restrict__ out) {
  constexpr int kPer = D / 32;  // output columns per lane
  constexpr int kEarly = 4;      // partitions whose rows are loaded before the length is known
  // the next launch of the stream may be scheduled now (it waits for this
  // grid's completion before touching memory)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= num_seqs * num_q_heads) return;
  const int b = row / num_q_heads;
  const int64_t base = static_cast<int64_t>(row) * max_parts;
  // one round of loads for the common case: the length, the (m, l) of
  // partitions lane, and the first kEarly partitions' rows of this lane's
  // columns (entries past the sequence's partitions are read from the
  // workspace, which is sized for max_parts, and ignored)
  int L = seq_lens[b];
  const bool lane_part = lane < max_parts;
  const float m_lane = lane_part ? part_m[base + lane] : -INFINITY;
  const float l_lane = lane_part ? part_l[base + lane] : 0.f;
  float early[kEarly][kPer];
#pragma unroll
  for (int t = 0; t < kEarly; ++t) {
    if (t < max_parts) {
      const float* o = part_o + (base + t) * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 x = *reinterpret_cast<const float4*>(o);
        early[t][0] = x.x; early[t][1] = x.y; early[t][2] = x.z; early[t][3] = x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(o);
        early[t][0] = x.x; early[t][1] = x.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < kPer; ++i) early[t][i] = 0.f;
    }
  }
  L = L < 0 ? 0 : (L > max_tokens ? max_tokens : L);
  if (L <= part_tokens) return;  // one partition: written by the decode kernel
  const int np = (L + part_tokens - 1) / part_tokens;
  float M = lane < np ? m_lane : -INFINITY;
  for (int q = lane + 32; q < np; q += 32) M = fmaxf(M, part_m[base + q]);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
  float den = 0.f;
  for (int q0 = 0; q0 < np; q0 += 32) {
    const int nq = min(32, np - q0);
    const float mq = q0 == 0 ? m_lane : (lane < nq ? part_m[base + q0 + lane] : -INFINITY);
    const float lq = q0 == 0 ? l_lane : (lane < nq ? part_l[base + q0 + lane] : 0.f);
    const float f_mine = lane < nq ? fast_exp2(mq - M) : 0.f;
    den += lane < nq ? f_mine * lq : 0.f;
    const float* o = part_o + (base + q0) * D + lane * kPer;
    int j = 0;
    if (q0 == 0) {  // the rows loaded up front
#pragma unroll
      for (int t = 0; t < kEarly; ++t) {
        const float f = __shfl_sync(kFull, f_mine, t);
        if (t < nq) {
#pragma unroll
          for (int i = 0; i < kPer; ++i) acc[i] += f * early[t][i];
        }
      }
      j = min(kEarly, nq);
    }
    for (; j + 4 <= nq; j += 4) {
      float v[4][kPer];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if constexpr (kPer == 4) {
          const float4 x = *reinterpret_cast<const float4*>(o + (j + t) * D);
          v[t][0] = x.x; v[t][1] = x.y; v[t][2] = x.z; v[t][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2*>(o + (j + t) * D);
          v[t][0] = x.x; v[t][1] = x.y;
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float f = __shfl_sync(kFull, f_mine, j + t);
#pragma unroll
        for (int i = 0; i < kPer; ++i) acc[i] += f * v[t][i];
      }
    }
    for (; j < nq; ++j) {
      const float f = __shfl_sync(kFull, f_mine, j);
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] += f * o[j * D + i];
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(kFull, den, o);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float* dst = out + static_cast<int64_t>(row) * D + lane * kPer;
#pragma unroll
  for (int i = 0; i < kPer; ++i) dst[i] = acc[i] * inv;
}

// ---------------------------------------------------------------------------
// merge for batches whose sequences can span more than 32 partitions (long
// contexts): one CTA per (sequence, query head), its 8 warps each merging a
// contiguous eighth of the partitions against their own max, then warp 0
// combining the 8 records (max, sum, row) the same way.  A warp per row
// walked the 256 partitions of a 128K-token sequence one after another.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) merge_wide_kernel(const int32_t* __restrict__ seq_lens, int32_t num_seqs,
                                                         int32_t num_q_heads, int32_t max_tokens, int32_t part_tokens,
                                                         int32_t max_parts, const float* __restrict__ part_m,
                                                         const float* __restrict__ part_l,
                                                         const float* __restrict__ part_o, float* __restrict__ out) {
  constexpr int kPer = D / 32;
  __shared__ float rec_m[8], rec_l[8];
  __shared__ float rec_o[8][D];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (row >= num_seqs * num_q_heads) return;
  int L = seq_lens[row / num_q_heads];
  L = L < 0 ? 0 : (L > max_tokens ? max_tokens : L);
  if (L <= part_tokens) return;  // one partition: written by the decode kernel (uniform over the CTA)
  const int np = (L + part_tokens - 1) / part_tokens;
  const int per = (np + 7) / 8, q0 = warp * per, q1 = min(np, q0 + per);  // this warp's partitions
  const int64_t base = static_cast<int64_t>(row) * max_parts;
  float M = -INFINITY;
  for (int q = q0 + lane; q < q1; q += 32) M = fmaxf(M, part_m[base + q]);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
  float den = 0.f;
  for (int g0 = q0; g0 < q1; g0 += 32) {
    const int nq = min(32, q1 - g0);
    const float f_mine = lane < nq ? fast_exp2(part_m[base + g0 + lane] - M) : 0.f;
    den += lane < nq ? f_mine * part_l[base + g0 + lane] : 0.f;
    const float* o = part_o + (base + g0) * D + lane * kPer;
    int j = 0;
    for (; j + 4 <= nq; j += 4) {
      float v[4][kPer];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
#pragma unroll
        for (int i = 0; i < kPer; ++i) v[t][i] = o[(j + t) * D + i];
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float f = __shfl_sync(kFull, f_mine, j + t);
#pragma unroll
        for (int i = 0; i < kPer; ++i) acc[i] += f * v[t][i];
      }
    }
    for (; j < nq; ++j) {
      const float f = __shfl_sync(kFull, f_mine, j);
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] += f * o[j * D + i];
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(kFull, den, o);
  if (lane == 0) {
    rec_m[warp] = M;  // -inf for a warp without partitions
    rec_l[warp] = den;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) rec_o[warp][lane * kPer + i] = acc[i];
  __syncthreads();
  if (warp != 0) return;
  float Mt = -INFINITY;
#pragma unroll
  for (int w = 0; w < 8; ++w) Mt = fmaxf(Mt, rec_m[w]);
  float res[kPer], dt = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) res[i] = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const float f = rec_m[w] == -INFINITY ? 0.f : fast_exp2(rec_m[w] - Mt);
    dt += f * rec_l[w];
#pragma unroll
    for (int i = 0; i < kPer; ++i) res[i] += f * rec_o[w][lane * kPer + i];
  }
  const float inv = dt > 0.f ? 1.f / dt : 0.f;
  float* dst = out + static_cast<int64_t>(row) * D + lane * kPer;
#pragma unroll
  for (int i = 0; i < kPer; ++i) dst[i] = res[i] * inv;
}

}  // namespace pkv
