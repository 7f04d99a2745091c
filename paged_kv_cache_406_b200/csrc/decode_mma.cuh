// PagedAttention decode on tensor cores, for 16-bit K/V with grouped-query
// heads (G = num_q_heads / num_kv_heads in {2, 4, 8}).
//
// Same work list, ring and merge as decode_kernel (decode.cuh); what changes
// is how a consumer warp turns a 16-token chunk into scores and outputs:
//
//   S^T[16 tokens][8 heads] = K[16][D] · Q^T[D][8]     (mma m16n8k16, D/16 steps)
//   O^T[D][8 heads]        += V^T[D][16] · P^T[16][8]  (mma m16n8k16, D/16 tiles)
//
// Query heads of one KV head fill the 8 columns (G of them real, the rest
// zero), so q·Kᵀ of a GQA group is a dense [tokens x dims] x [dims x heads]
// product.  P is rounded to a pair of 16-bit values hi + lo (two mmas) so the
// weights keep about 16 significant bits; accumulation is fp32.
//
// K and V chunks arrive by 3-D tensor-map TMA loads (one per block and per K
// or V: all 128-byte column halves of br rows) with 128-byte swizzle (16-byte
// chunk c of row r is stored at chunk c ^ (r mod 8)), so the ldmatrix reads of
// 8 consecutive rows hit 8 different bank groups.  A chunk
// is 16 tokens: one block (block_size 16), two blocks (8) or half a block (32).
// Token rows past the end of the sequence are masked out of the softmax and
// their V rows are zeroed in shared memory before the P·V product, so stale
// pool contents (possibly NaN) never reach the accumulators.
#pragma once

#include <cuda.h>
#include <cuda_fp8.h>

#include "decode.cuh"

namespace pkv {

constexpr int kChunkTokens = 16;
// Two producer warps share the issuing: warp kConsumerWarps + pr issues the
// chunks whose CTA-wide index has parity pr (the ring stages of that parity).
// One lane issuing every TMA load (~150 cycles each plus its bookkeeping) was
// the measured limit of the single-producer kernel.
constexpr int kMmaProducers = 2;
constexpr int kMmaThreads = (kConsumerWarps + kMmaProducers) * 32;


template <int D>
struct MmaLayout {
  static constexpr int kHalves = D / 64;                   // 128-byte column halves of a 16-bit row
  static constexpr int kTileBytes = kChunkTokens * D * 2;  // 16-token K (or V) chunk
  static constexpr int kStageBytes = 2 * kTileBytes;
};

template <typename T, int D, int G>
struct MmaSmem {
  using L = MmaLayout<D>;
  static constexpr int kCW = kConsumerWarps;
  static constexpr int kThreads = kMmaThreads;
  static constexpr int kMergeFloats = G * D + 2 * G;
  __host__ __device__ static size_t ring_bytes(int ns) {
    return size_t(ns) * L::kStageBytes;
  }
  __host__ __device__ static size_t bytes(int ns) {
    // + 1024: the dynamic shared memory base is aligned up to the 1024-byte swizzle atom
    return 1024 + ring_bytes(ns) + 2 * kCW * kMergeFloats * sizeof(float) + 2 * ns * sizeof(uint64_t) + 16 +
           kMmaProducers * 128;
  }
};

// A chunk tile in shared memory is built from TMA boxes of `br` rows (br = 16,
// or 8 when block_size is 8 and a chunk spans two blocks).  Each box holds,
// for every 128-byte column half h, br rows of 128 B with the 128-byte
// swizzle (16-byte chunk c of row r at chunk position c ^ (r mod 8)):
//     byte offset of (row r, half h) = (r / br) * (halves * br * 128) + h * br * 128 + (r % br) * 128
__device__ __forceinline__ uint32_t row_offset(int r, int h, int br_shift, int halves) {
  const int br = 1 << br_shift;
  return static_cast<uint32_t>(((r >> br_shift) * halves * br + h * br + (r & (br - 1))) * 128);
}

// Tensor maps of the K and V pools of a batch (pool c: k[c], v[c]).
struct PoolMaps {
  CUtensorMap k[kMaxPools];
  CUtensorMap v[kMaxPools];
};

// Block size of a pool as shifts: log2(block_size) and log2(rows per TMA box)
// (8 rows for 8-token blocks, else 16: a 16-token chunk is one box, two
// boxes of 8-token blocks, or half a 32-token block).
__device__ __forceinline__ int bs_shift_of(int bs) { return bs == 8 ? 3 : (bs == 16 ? 4 : 5); }
__device__ __forceinline__ int br_shift_of(int bs) { return bs == 8 ? 3 : 4; }

// Two CTAs fit an SM (shared memory); declaring it lets the compiler use up
// to 170 registers (146 for head_dim 128) instead of its own choice of 96,
// which was 1-2 % slower.
// kMulti: the batch spans up to kMaxPools pools of different block sizes
// (each work unit reads its sequence's pool); otherwise pool 0 only.
// kStall: the instance that honours DecodeParams::stall_cta (the test of the
// bounded waits); production launches use the instance without the check.
template <typename T, int D, int G, bool kMulti = false, bool kStall = false>
__global__ void __launch_bounds__(kMmaThreads, 2)
    decode_mma_kernel(const DecodeParams p, const __grid_constant__ PoolMaps maps) {
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  using L = MmaLayout<D>;
  constexpr int kCW = kConsumerWarps;
  constexpr int kSteps = D / 16;  // k-steps of q·Kᵀ and m-tiles of P·V
  constexpr int kHalves = L::kHalves;
  constexpr int kMF = MmaSmem<T, D, G>::kMergeFloats;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int NS = p.n_stages;
  float* merge = reinterpret_cast<float*>(smem + MmaSmem<T, D, G>::ring_bytes(NS));
  uint64_t* full = reinterpret_cast<uint64_t*>(merge + 2 * kCW * kMF);
  uint64_t* empty = full + NS;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NS);
  int32_t* tab = reinterpret_cast<int32_t*>(empty + NS) + 4;  // 32 block-table entries per producer
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

  if (warp >= kCW) {
    // ----------------------------- producers -----------------------------
    // Both producer warps walk every unit and refill their own 32-entry
    // block-table window; lane 0 of producer pr alone issues the window's
    // chunks of parity pr, so the per-chunk path has no warp-wide
    // synchronisation.
    const int pr = warp - kCW;
    int32_t* mytab = tab + 32 * pr;
    if (lane < (kMulti ? p.n_pools : 1)) {
      prefetch_tensormap(&maps.k[lane]);
      prefetch_tensormap(&maps.v[lane]);
    }
    const uint64_t policy = l2_evict_first_policy();
    const uint64_t tab_policy = l2_evict_last_policy();
    int s = pr;           // this producer's stages: pr, pr + 2, ...
    uint32_t ph = 0, issued = 0, skipped = 0;  // stage uses so far; the first `skipped` of them issued no copy
    uint32_t cg = 0;      // CTA-wide chunk index of the unit's first chunk
    bool ok = true;
    for (int r = 0, w = unit_index(0); w < n_work && ok; w = unit_index(++r)) {
      const bool stall = kStall && r == 0 && p.stall_cta == static_cast<int>(blockIdx.x);
      const WorkUnit u = load_unit<kMulti>(p, w);
      const PoolView pv = kMulti ? pick3(p.pool, u.c) : p.pool[0];
      const int BS = pv.block_size, bs_shift = bs_shift_of(BS), br_shift = br_shift_of(BS);
      const uint32_t box_bytes = (1u << br_shift) * D * 2;               // one K (or V) box
      const uint32_t blk_off = L::kHalves * (1u << br_shift) * 128;  // second box of a chunk (block_size 8)
      const CUtensorMap* tmap_k = &maps.k[kMulti ? u.c : 0];
      const CUtensorMap* tmap_v = &maps.v[kMulti ? u.c : 0];
      const int32_t* trow = pv.tables + static_cast<int64_t>(u.b - pv.seq0) * pv.max_blocks + (u.t0 >> bs_shift);
      const int nch = (u.t1 - u.t0 + kChunkTokens - 1) / kChunkTokens;
      const int ybase = u.g * BS;
      for (int wb = 0; wb < u.nblk && ok; wb += 32) {
        mytab[lane] = wb + lane < u.nblk ? ld_table(trow + wb + lane, tab_policy) : 0;
        __syncwarp();
        if (lane == 0) {
          const int k_begin = (wb << bs_shift) >> 4;
          const int k_end = min(nch, ((wb + 32) << bs_shift) >> 4);
          for (int k = k_begin + ((pr - static_cast<int>(cg) - k_begin) & 1); k < k_end; k += kMmaProducers) {
            if (!mbar_wait(smem_addr(empty + s), ph ^ 1, abort_flag)) {
              record_error(PKV_ERR_DEVICE_TIMEOUT);
              *abort_flag = 1;
              ok = false;
              break;
            }
            const int jb = (k << 4) >> bs_shift;  // unit-relative block of the chunk
            const int nb_here = BS == 8 ? min(2, u.nblk - jb) : 1;
            const int row0 = BS == 32 ? (k & 1) << 4 : 0;
            const uint32_t bar = smem_addr(full + s);
            const uint32_t kdst = ring_s + s * L::kStageBytes;
            if (!stall) mbar_arrive_expect_tx(bar, nb_here * 2 * box_bytes);
            else ++skipped;  // nothing will land in this stage: its consumer's wait runs out
            for (int i = 0; i < nb_here && !stall; ++i) {
              int phys = mytab[jb - wb + i];
              if (static_cast<unsigned>(phys) >= static_cast<unsigned>(pv.num_blocks)) {
                record_error(PKV_ERR_BAD_BLOCK);
                phys = 0;
              }
              const int32_t y = phys * p.num_kv_heads * BS + ybase + row0;
              tma_load_3d(kdst + i * blk_off, tmap_k, 0, y, 0, bar, policy);
              tma_load_3d(kdst + L::kTileBytes + i * blk_off, tmap_v, 0, y, 0, bar, policy);
            }
            ++issued;
            s += kMmaProducers;
            if (s >= NS) {
              s -= NS;
              ph ^= 1;
            }
          }
        }
        __syncwarp();
        ok = __shfl_sync(kFull, ok, 0);
      }
      cg += nch;
    }
    // No copy may still be landing in shared memory when the CTA exits: wait
    // (bounded) for the last phase issued into each of this producer's stages.
    if (lane == 0) {
      const int mine = NS / kMmaProducers;  // stages pr, pr + 2, ...
      for (int j = 0; j < mine && j < static_cast<int>(issued); ++j) {
        const uint32_t uses = (issued - j + mine - 1) / mine;
        if (j + mine * (uses - 1) < skipped) continue;  // its last use carried no copy
        const int st = pr + kMmaProducers * j;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(smem_addr(full + st), (uses - 1) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    return;
  }

  // ------------------------------ consumers ------------------------------
  const int gq = lane >> 2;  // fragment row group: token (S^T) / dim (O^T) / head (B operands)
  const int tq = lane & 3;   // fragment column pair: heads 2tq, 2tq+1
  // ldmatrix row addresses of this lane: K chunk (A operand) and V chunk (A = Vᵀ via .trans)
  const int ra = (lane & 7) + ((lane >> 3) & 1) * 8, ca = lane >> 4;
  const int rv = (lane & 7) + (lane >> 4) * 8, cv = (lane >> 3) & 1;
  const int xa = ra & 7, xv = rv & 7;
  const int src0 = 4 * (2 * tq) + (gq >> 1), src1 = src0 + 4;  // Pᵀ transpose sources
  const uint32_t sel = (gq & 1) ? 0x7632u : 0x5410u;
  const float sl = p.scale_log2;
  uint32_t c = 0;
  int iter = 0;
  bool ok = true;
  for (int w = unit_index(0); w < n_work; w = unit_index(++iter)) {
    const WorkUnit u = load_unit<kMulti>(p, w);
    const int nch = (u.t1 - u.t0 + kChunkTokens - 1) / kChunkTokens;
    // 16-bit pools: the MMAs read the ring chunk itself, built from boxes of
    // br rows (the unit's pool decides br)
    const int tile_shift = br_shift_of(kMulti ? pick3(p.pool, u.c).block_size : p.pool[0].block_size);
    uint32_t offa[kHalves], offv[kHalves];
#pragma unroll
    for (int h = 0; h < kHalves; ++h) {
      offa[h] = row_offset(ra, h, tile_shift, kHalves);
      offv[h] = row_offset(rv, h, tile_shift, kHalves);
    }

    // B fragments of Qᵀ: column n = head gq (zero for the padding heads >= G)
    uint32_t qb[kSteps][2];
    {
      const T* qrow = static_cast<const T*>(p.q) + (static_cast<int64_t>(u.b) * p.num_q_heads + u.g * G + gq) * D;
#pragma unroll
      for (int ks = 0; ks < kSteps; ++ks) {
        qb[ks][0] = gq < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tq)) : 0u;
        qb[ks][1] = gq < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tq + 8)) : 0u;
      }
    }
    float acc[kSteps][4];
#pragma unroll
    for (int mt = 0; mt < kSteps; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2tq, 2tq+1

    const int k0 = (warp - static_cast<int>(c % kCW) + kCW) % kCW;
    int s = (c + k0) % NS;
    uint32_t ph = ((c + k0) / NS) & 1;
    for (int k = k0; k < nch && ok; k += kCW) {
      const bool landed = __all_sync(kFull, mbar_wait(smem_addr(full + s), ph, abort_flag));
      if (!landed) {
        if (lane == 0) {
          record_error(PKV_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
        }
        ok = false;
        break;
      }
      uint32_t kbase = ring_s + s * L::kStageBytes;
      uint32_t vbase = kbase + L::kTileBytes;
      const int nv = min(kChunkTokens, u.t1 - (u.t0 + k * kChunkTokens));
      // ---- scores: S^T = K · Qᵀ ----
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < kSteps; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(kbase + offa[ks / 4] + (((2 * (ks % 4) + ca) ^ xa) << 4), a);
        mma_16816<T>(sc, a, qb[ks][0], qb[ks][1]);
      }
      const bool v0 = gq < nv, v1 = gq + 8 < nv;  // tokens gq and gq + 8 of the chunk
      const float s0 = v0 ? sc[0] * sl : -INFINITY, s1 = v0 ? sc[1] * sl : -INFINITY;
      const float s2 = v1 ? sc[2] * sl : -INFINITY, s3 = v1 ? sc[3] * sl : -INFINITY;

      // ---- online softmax (the running max moves only by more than the threshold) ----
      float bm0 = fmaxf(s0, s2), bm1 = fmaxf(s1, s3);
      if (__any_sync(kFull, bm0 > m0 + kRescaleThreshold || bm1 > m1 + kRescaleThreshold)) {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          bm0 = fmaxf(bm0, __shfl_xor_sync(kFull, bm0, o));
          bm1 = fmaxf(bm1, __shfl_xor_sync(kFull, bm1, o));
        }
        const float n0 = fmaxf(m0, bm0), n1 = fmaxf(m1, bm1);
        const float f0 = n0 == -INFINITY ? 1.f : fast_exp2(m0 - n0);
        const float f1 = n1 == -INFINITY ? 1.f : fast_exp2(m1 - n1);
#pragma unroll
        for (int mt = 0; mt < kSteps; ++mt) {
          acc[mt][0] *= f0;
          acc[mt][2] *= f0;
          acc[mt][1] *= f1;
          acc[mt][3] *= f1;
        }
        l0 *= f0;
        l1 *= f1;
        m0 = n0;
        m1 = n1;
      }
      const float p0 = fast_exp2(s0 - m0), p1 = fast_exp2(s1 - m1);
      const float p2 = fast_exp2(s2 - m0), p3 = fast_exp2(s3 - m1);
      l0 += p0 + p2;
      l1 += p1 + p3;

      // ---- P as hi + lo 16-bit pairs, transposed into B fragments of Pᵀ ----
      uint32_t ha, la, hb, lb;
      split_pack<T>(p0, p1, ha, la);  // token gq:     heads 2tq, 2tq+1
      split_pack<T>(p2, p3, hb, lb);  // token gq + 8
      const uint32_t bh0 = __byte_perm(__shfl_sync(kFull, ha, src0), __shfl_sync(kFull, ha, src1), sel);
      const uint32_t bh1 = __byte_perm(__shfl_sync(kFull, hb, src0), __shfl_sync(kFull, hb, src1), sel);
      const uint32_t bl0 = __byte_perm(__shfl_sync(kFull, la, src0), __shfl_sync(kFull, la, src1), sel);
      const uint32_t bl1 = __byte_perm(__shfl_sync(kFull, lb, src0), __shfl_sync(kFull, lb, src1), sel);

      // ---- rows past the sequence end: zero V so stale values cannot reach P·V ----
      if (nv < kChunkTokens) {
        const int per_row = 8 * kHalves;
        const int total = (kChunkTokens - nv) * per_row;
        for (int i = lane; i < total; i += 32) {
          const int row = nv + i / per_row, rem = i % per_row;
          const uint32_t addr = vbase + row_offset(row, rem / 8, tile_shift, kHalves) + (rem % 8) * 16;
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
        }
        __syncwarp();
      }

      // ---- O^T += V^T · P^T ----
#pragma unroll
      for (int mt = 0; mt < kSteps; ++mt) {
        uint32_t a[4];
        ldmatrix_x4_trans(vbase + offv[mt / 4] + (((2 * (mt % 4) + cv) ^ xv) << 4), a);
        mma_16816<T>(acc[mt], a, bh0, bh1);
        mma_16816<T>(acc[mt], a, bl0, bl1);
      }
      if (nv < kChunkTokens) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(empty + s));
      s += kCW;
      if (s >= NS) {
        s -= NS;
        ph ^= 1;
      }
    }
    c += nch;

    // ---- publish this warp's record, then merge the warps ----
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(kFull, l0, o);
      l1 += __shfl_xor_sync(kFull, l1, o);
    }
    float* mb = merge + ((iter & 1) * kCW + warp) * kMF;
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
#pragma unroll
    for (int mt = 0; mt < kSteps; ++mt) {
      // fragment rows gq and gq + 8 of m-tile mt: dims d and d + dd
      const int d = 16 * mt + gq;
      if (h0 < G) {
        mb[h0 * D + d] = acc[mt][0];
        mb[h0 * D + d + 8] = acc[mt][2];
      }
      if (h1 < G) {
        mb[h1 * D + d] = acc[mt][1];
        mb[h1 * D + d + 8] = acc[mt][3];
      }
    }
    if (gq == 0) {
      if (h0 < G) {
        mb[G * D + h0] = m0;
        mb[G * D + G + h0] = l0;
      }
      if (h1 < G) {
        mb[G * D + h1] = m1;
        mb[G * D + G + h1] = l1;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
    merge_store<G, D, kCW>(merge + (iter & 1) * kCW * kMF, u, p);
  }
}

}  // namespace pkv
