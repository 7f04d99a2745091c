// Paged decode attention over e4m3 (FP8) K/V pools on the fifth-generation
// tensor cores: tcgen05.mma kind::f8f6f4 reads the e4m3 codes straight from
// the shared-memory tiles TMA wrote, so no code is ever widened in registers.
//
// vLLM paging page §3 phase 2 defines the computation (gather the sequence's
// blocks, q·Kᵀ, softmax, ·V); the overview page §5.1 stores K and V as FP8
// (read here as e4m3 codes times one fp32 scale per pool).  The result is the
// attention of the dequantised cache, as the 16-bit kernels compute it.
//
// Per CTA (persistent, two per SM) and per work unit (sequence, partition,
// KV head, as planned by plan_body), in chunks of 128 tokens:
//   producer warp   TMA: the chunk's K and V rows (128 B each) into a 3-stage
//                   ring with the 128-byte swizzle, one box per 16 (or 8) rows
//   MMA warp        S^T[tok][n] = K[tok][:] · Qt[n][:]   (M 128, N 8..24)
//                   O^T[d][n]  += V[:, d]ᵀ · Pt[:, n]     (M 128, N 16..32)
//                   V read MN-major from the same tile layout; D in tensor memory
//   softmax warps   thread t owns token t of S^T and dim t of O^T
//
// e4m3 MMAs take e4m3 operands on both sides, so q and P enter as sums of
// e4m3 terms, each term a separate column block of N (its own accumulator):
//   q:  x0 = q·c (c a power of two putting max|q| in [128, 256)); term i =
//       e4m3(x_i), x_{i+1} = 16·(x_i - term i).  Three terms hold an f16 q
//       exactly (4 significant bits a term; f16 has 11) but for elements
//       below 2^-15 of the head's largest, which stay within 2^-24 of it; S
//       is the dot product summed in fp32: S = (col0 + col1/16 + col2/256) / c.
//   P:  P = 2^(s - m) <= 2^8 split the same way into four terms (about 16
//       significant bits); O = col0 + col1/16 + col2/256 + col3/4096.  Three
//       terms (12 bits) miss the output tolerance over full-range codes.
// The tensor cores accumulate these products to fp32 precision.
//
// The running max m of each head moves only when a chunk's max passes it by
// more than 2^8 (the threshold of the 16-bit kernels); then O (in tensor
// memory) and the row sums are rescaled once.  Rows past the sequence end:
// their scores are -inf and their V rows are zeroed before P·V reads them.
#pragma once

#include <cuda_fp8.h>

#include "decode.cuh"
#include "device_common.cuh"
#include "tcgen05.cuh"

namespace pkv {
namespace t8 {

constexpr int kTok = 128;     // tokens per chunk: M of S^T, contraction of P·V
constexpr int kD = 128;       // head_dim: one 128-byte e4m3 row
constexpr int kTermsQ = 3;
constexpr int kTermsP = 4;
constexpr int kProducer = 4, kMmaWarp = 5;
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = kTok * kD;        // one chunk of K (or V)
constexpr uint32_t kStageBytes = 2 * kTileBytes;  // K then V
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColS = 0, kColO = 64;  // S^T buffers at columns 0 and 32, O^T at 64
constexpr float kThreshold = 8.0f;

// N of the two MMAs: terms x heads, rounded up to the shape rules
__host__ __device__ constexpr int n_s(int g) { return (kTermsQ * g + 7) / 8 * 8; }
__host__ __device__ constexpr int n_o(int g) { return (kTermsP * g + 15) / 16 * 16; }

// shared memory (from a 1024-byte aligned base) for a ring of NSt stages and
// G query heads per KV head
template <int NSt, int G>
struct Layout {
  static constexpr uint32_t kPBuf = n_o(G) / 16 * 2048;  // P terms of one chunk: [group][token][16 B]
  static constexpr uint32_t kOffQ = NSt * kStageBytes;   // q terms: n_s(G) rows x 128 B, swizzled
  static constexpr uint32_t kQBytes = n_s(G) / 8 * 1024;
  static constexpr uint32_t kOffP = kOffQ + kQBytes;     // two P-terms buffers
  static constexpr uint32_t kOffRed = kOffP + 2 * kPBuf;  // [3][4 warps][8 heads]: chunk maxima (2), row sums
  static constexpr uint32_t kOffQs = kOffRed + 3 * 4 * 8 * 4;
  static constexpr uint32_t kOffBar = kOffQs + 8 * 4;
  enum : int { kBFull = 0, kBEmpty = kBFull + NSt, kBQFull = kBEmpty + NSt, kBSFull = kBQFull + 1,
               kBSFree = kBSFull + 2, kBPFull = kBSFree + 2, kBPFree = kBPFull + 2, kBDrain = kBPFree + 2,
               kNumBars = kBDrain + 1 };
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // abort flag, tensor-memory address
  static constexpr size_t kSmemBytes = kOffMisc + 16 + 1024;   // + alignment slack
  // arrivals per phase: the q-full, S-free and P-full barriers take all 128
  // softmax threads; the rest one arrival (a TMA expect or an MMA commit)
  __host__ __device__ static constexpr uint32_t bar_count(int i) {
    return (i == kBQFull || i == kBSFree || i == kBSFree + 1 || i == kBPFull || i == kBPFull + 1) ? 128u : 1u;
  }
};

// Named barrier 1 over the four softmax warps, returning whether any thread
// passed `v` true (the warps leave a loop together when one of them failed).
__device__ __forceinline__ bool softmax_bar_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, 1, 128, q;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// A softmax thread gave up waiting: the error is recorded and every other
// role's waits end at once.
__device__ __forceinline__ void abort_softmax_impl(volatile int* abort_flag) {
  if (threadIdx.x == 0) {
    record_error(PKV_ERR_DEVICE_TIMEOUT);
    *abort_flag = 1;
  }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Reduce-scatter of G per-lane values over the warp: lane l returns the
// reduction (max, or sum) of head (l >> (5 - log2 G)) over all 32 lanes.
// The first log2 G steps halve each lane's list (the half a lane keeps is
// chosen by its lane bit), so G heads cost 5 + G - 1 - log2 G shuffles
// (6 for G = 4) instead of 5 G.
template <int G, bool kMax>
__device__ __forceinline__ float reduce_scatter(const float (&v)[G], int lane) {
  float a[G];
#pragma unroll
  for (int i = 0; i < G; ++i) a[i] = v[i];
  int o = 16;
#pragma unroll
  for (int n = G; n > 1; n >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float keep = up ? a[i + n / 2] : a[i], give = up ? a[i] : a[i + n / 2];
      const float other = __shfl_xor_sync(0xffffffffu, give, o);
      a[i] = kMax ? fmaxf(keep, other) : keep + other;
    }
  }
#pragma unroll
  for (; o > 0; o >>= 1) {
    const float other = __shfl_xor_sync(0xffffffffu, a[0], o);
    a[0] = kMax ? fmaxf(a[0], other) : a[0] + other;
  }
  return a[0];
}

// The head whose reduction lane l holds after reduce_scatter<G>, and whether
// l is the first lane holding it.
template <int G>
__device__ __forceinline__ int scatter_head(int lane) {
  return G == 1 ? 0 : (lane >> (G == 2 ? 4 : (G == 4 ? 3 : 2))) & (G - 1);
}
template <int G>
__device__ __forceinline__ bool scatter_first(int lane) {
  return (lane & (32 / G - 1)) == 0;
}

// Two fp32 values rounded to e4m3 (nearest, ties to even; no value here
// exceeds 448), x0 in the low byte; and the two codes' values.
__device__ __forceinline__ uint32_t e4m3_pair(float x0, float x1, float& d0, float& d1) {
  const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(c, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  d0 = f.x;
  d1 = f.y;
  return static_cast<uint32_t>(c);
}

}  // namespace t8

// kStall: the instance that honours DecodeParams::stall_cta (the test of the
// bounded waits: that CTA's producer issues no copy for its first work unit);
// production launches use the instance without the check.
template <int G, int NSt, bool kStall = false>
__global__ void __launch_bounds__(t8::kThreads, NSt <= 2 ? 3 : (NSt == 3 ? 2 : 1))
    decode_tc8_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v) {
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  constexpr int NS_ = t8::n_s(G), NO = t8::n_o(G);
  using L = t8::Layout<NSt, G>;
  static_assert(NS_ <= 32 && NO <= 32, "S^T and O^T columns");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t base = smem_addr(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc + 4);
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);
  float* qs = reinterpret_cast<float*>(smem + L::kOffQs);
  auto bar = [&](int i) { return base + L::kOffBar + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bar(i), L::bar_count(i));
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp < 4) {
    // q-term rows past kTermsQ * G are never written: zero them (and the rest) once
    uint4* q = reinterpret_cast<uint4*>(smem + L::kOffQ);
    for (int i = threadIdx.x; i < static_cast<int>(L::kQBytes) / 16; i += 128) q[i] = make_uint4(0u, 0u, 0u, 0u);
    uint4* pz = reinterpret_cast<uint4*>(smem + L::kOffP);
    for (int i = threadIdx.x; i < 2 * static_cast<int>(L::kPBuf) / 16; i += 128) pz[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (warp == t8::kMmaWarp) {
    tc::tmem_alloc(smem_addr(tmem_slot), t8::kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == t8::kProducer && lane == 0) {
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  asm volatile("griddepcontrol.wait;" ::: "memory");               // the plan (and append) are complete
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // let merge_kernel be scheduled

  const int n_work = *p.n_items * p.num_kv_heads;
  const PoolView pv = p.pool[0];
  const int BS = pv.block_size;
  const int box_rows = BS < 16 ? BS : 16;  // TMA box: 16 rows (8 for block size 8), 16-token aligned

  if (warp == t8::kProducer) {
    // ------------------------------- TMA producer -------------------------------
    // Lane i issues box i of each chunk.  The block-table entries of a unit
    // come from a 32-entry window (lane i holds entry wb + i, counted from
    // the unit's first block), and the next unit's work item and first
    // window are loaded one unit ahead, so no chunk waits on a table load.
    const uint64_t policy = l2_evict_first_policy();
    const uint64_t tab_policy = l2_evict_last_policy();
    auto table_entry = [&](const WorkUnit& uu, int kb) -> int32_t {  // block kb of the unit, or 0 past its end
      const int b0 = uu.t0 / BS, nb = (uu.t1 - 1) / BS - b0 + 1;
      return kb < nb ? ld_table(pv.tables + static_cast<int64_t>(uu.b) * pv.max_blocks + b0 + kb, tab_policy) : 0;
    };
    WorkUnit un{};
    int32_t tab_n = 0;
    auto prefetch = [&](int wn) {
      if (wn >= n_work) return;
      un = load_unit<false>(p, wn);
      tab_n = un.t1 > un.t0 ? table_entry(un, lane) : 0;
    };
    prefetch(unit_index(0));
    bool ok = true;
    int j = 0, skipped = 0;  // ring uses so far; the first `skipped` of them carried no copy
    for (int r = 0, w = unit_index(0); w < n_work && ok; w = unit_index(++r)) {
      const bool stall = kStall && r == 0 && p.stall_cta == static_cast<int>(blockIdx.x);
      const WorkUnit u = un;
      int32_t tab = tab_n;
      int wb = 0;
      prefetch(unit_index(r + 1));
      const int nc = (u.t1 - u.t0 + t8::kTok - 1) / t8::kTok;
      const int b0 = u.t0 / BS;
      for (int c = 0; c < nc; ++c) {
        const int s = j % NSt;
        const int a = u.t0 + c * t8::kTok;
        const int nbox = (min(t8::kTok, u.t1 - a) + box_rows - 1) / box_rows;
        const int kb_first = a / BS - b0, kb_last = (min(a + t8::kTok, u.t1) - 1) / BS - b0;
        if (kb_last >= wb + 32) {  // the chunk's blocks lie past the window: move it to the chunk
          wb = kb_first;
          tab = table_entry(u, wb + lane);
        }
        const int tok = a + lane * box_rows;  // first token of box `lane`
        int phys = __shfl_sync(0xffffffffu, tab, (min(tok, u.t1 - 1) / BS - b0 - wb) & 31);
        int32_t y = 0;
        if (lane < nbox) {
          if (static_cast<unsigned>(phys) >= static_cast<unsigned>(pv.num_blocks)) {
            record_error(PKV_ERR_BAD_BLOCK);
            phys = 0;
          }
          y = (phys * p.num_kv_heads + u.g) * BS + tok % BS;
        }
        ok = __shfl_sync(0xffffffffu,
                         lane == 0 ? mbar_wait_sleep(bar(L::kBEmpty + s), ((j / NSt) & 1) ^ 1, abort_flag)
                                   : true,
                         0);
        if (!ok) break;
        if (stall) {  // nothing lands in this stage: the MMA warp's wait for it runs out
          ++skipped;
          ++j;
          continue;
        }
        if (lane == 0) mbar_arrive_expect_tx(bar(L::kBFull + s), static_cast<uint32_t>(nbox * box_rows * t8::kD * 2));
        __syncwarp();
        if (lane < nbox) {
          const uint32_t dst = base + s * t8::kStageBytes + static_cast<uint32_t>(lane * box_rows * t8::kD);
          tma_load_3d(dst, &tmap_k, 0, y, 0, bar(L::kBFull + s), policy);
          tma_load_3d(dst + t8::kTileBytes, &tmap_v, 0, y, 0, bar(L::kBFull + s), policy);
        }
        ++j;
      }
    }
    if (lane == 0) {
      if (!ok) {
        record_error(PKV_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
      }
      // no copy may still be landing when the CTA exits: the last fill of each stage
      for (int s = 0; s < NSt && s < j; ++s) {
        const int last = s + (j - 1 - s) / NSt * NSt;
        if (last < skipped) continue;  // its last use carried no copy
        mbar_drain(bar(L::kBFull + s), (last / NSt) & 1);
      }
    }
    __syncwarp();
  } else if (warp == t8::kMmaWarp) {
    // -------------------------------- MMA issuer --------------------------------
    constexpr uint32_t id_s = tc::idesc_e4m3(false, false, 128, NS_);
    constexpr uint32_t id_o = tc::idesc_e4m3(true, true, 128, NO);
    bool ok = true;
    int j = 0, uq = 0;  // chunks and (non-empty) units done
    for (int r = 0, w = unit_index(0); w < n_work && ok; w = unit_index(++r)) {
      const WorkUnit u = load_unit<false>(p, w);
      const int nc = (u.t1 - u.t0 + t8::kTok - 1) / t8::kTok;
      if (nc == 0) continue;
      if (lane == 0) {
        // S^T of chunk jj: K tile (K-major) times the q terms (K-major), 4 x 32 dims
        auto issue_s = [&](int jj) -> bool {
          const int s = jj % NSt;
          if (!mbar_wait_sleep(bar(L::kBFull + s), (jj / NSt) & 1, abort_flag)) return false;
          if (!mbar_wait_sleep(bar(L::kBSFree + (jj & 1)), ((jj >> 1) & 1) ^ 1, abort_flag)) return false;
          tc::fence_after_sync();
          const uint32_t kst = base + s * t8::kStageBytes;
#pragma unroll
          for (int ks = 0; ks < t8::kD / 32; ++ks) {
            tc::mma_e4m3_ss(tmem + t8::kColS + (jj & 1) * 32, tc::sw128_desc(kst + 32 * ks, 16, 1024),
                            tc::sw128_desc(base + L::kOffQ + 32 * ks, 16, 1024), id_s, ks > 0 ? 1u : 0u);
          }
          tc::commit(bar(L::kBSFull + (jj & 1)));
          return true;
        };
        ok = mbar_wait_sleep(bar(L::kBQFull), uq & 1, abort_flag) && issue_s(j);
        for (int c = 0; c < nc && ok; ++c) {
          const int jj = j + c;
          // The next chunk's scores go first when its tiles have landed (the
          // softmax warps then have work while this chunk's P·V runs);
          // otherwise this chunk's P·V goes first, so that its ring stage is
          // not held while the next chunk is still loading.
          bool next = c + 1 < nc;
          if (next && mbar_try_wait(bar(L::kBFull + (jj + 1) % NSt), ((jj + 1) / NSt) & 1)) {
            ok = issue_s(jj + 1);
            next = false;
          }
          if (!ok) break;
          ok = mbar_wait_sleep(bar(L::kBPFull + (jj & 1)), (jj >> 1) & 1, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          // O^T += V^T (MN-major: V rows as stored) · P terms (MN-major, 16-byte token rows), 4 x 32 tokens
          const uint32_t vst = base + (jj % NSt) * t8::kStageBytes + t8::kTileBytes;
          const uint32_t pb = base + L::kOffP + (jj & 1) * L::kPBuf;
#pragma unroll
          for (int ks = 0; ks < t8::kTok / 32; ++ks) {
            tc::mma_e4m3_ss(tmem + t8::kColO, tc::sw128_desc(vst + 4096 * ks, 16, 1024),
                            tc::smem_desc(pb + 512 * ks, 128, 2048, tc::kLayoutNone), id_o,
                            (c > 0 || ks > 0) ? 1u : 0u);
          }
          tc::commit(bar(L::kBEmpty + jj % NSt));
          tc::commit(bar(L::kBPFree + (jj & 1)));
          if (next) ok = issue_s(jj + 1);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      j += nc;
      ++uq;
    }
    if (lane == 0) {
      if (!ok) {
        record_error(PKV_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
      }
      // every MMA issued completes before tensor memory is freed
      tc::commit(bar(L::kBDrain));
      mbar_drain(bar(L::kBDrain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------- softmax warps -------------------------------
    const int t = threadIdx.x;  // token t of a chunk's S^T; dim t of O^T
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    unsigned char* qbuf = smem + L::kOffQ;
    bool fail = false;
    int j = 0;
    // Warp w writes the q terms of heads w, w + 4 (G >= 4; head w % G
    // otherwise), lane l dims 4l .. 4l+3.  The next unit's work item and q
    // words are loaded one unit ahead.
    constexpr int kHeadsPerWarp = G >= 4 ? G / 4 : 1;
    auto q_head = [&](int k) { return G >= 4 ? warp + 4 * k : warp % G; };
    WorkUnit un{};
    uint2 qn[kHeadsPerWarp];
    auto prefetch = [&](int wn) {
      if (wn >= n_work) return;
      un = load_unit<false>(p, wn);
      const int64_t r0 = static_cast<int64_t>(un.b) * p.num_q_heads + un.g * G;
#pragma unroll
      for (int k = 0; k < kHeadsPerWarp; ++k) {
        qn[k] = __ldg(reinterpret_cast<const uint2*>(static_cast<const __half*>(p.q) + (r0 + q_head(k)) * t8::kD +
                                                     4 * lane));
      }
    };
    prefetch(unit_index(0));
    for (int r = 0, w = unit_index(0); w < n_work; w = unit_index(++r)) {
      const WorkUnit u = un;
      uint2 qraw[kHeadsPerWarp];
#pragma unroll
      for (int k = 0; k < kHeadsPerWarp; ++k) qraw[k] = qn[k];
      prefetch(unit_index(r + 1));
      const int nc = (u.t1 - u.t0 + t8::kTok - 1) / t8::kTok;
      const int64_t row0 = static_cast<int64_t>(u.b) * p.num_q_heads + u.g * G;  // first query head row
      if (nc == 0) {  // an empty sequence (one partition): zeros
#pragma unroll
        for (int h = 0; h < G; ++h) p.out[(row0 + h) * t8::kD + t] = 0.f;
        continue;
      }

      // ---- q as three e4m3 terms: rows i*G + h of the swizzled B tile ----
      {
#pragma unroll
        for (int k = 0; k < kHeadsPerWarp; ++k) {
          const int h = q_head(k);
          const uint2 raw = qraw[k];
          const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
          const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
          float x[4] = {f01.x, f01.y, f23.x, f23.y};
          const float mx = t8::warp_max(fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))));
          const int e = mx > 0.f ? static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127 : 0;
          const float c = __uint_as_float(static_cast<uint32_t>(127 + 7 - e) << 23);  // max|q|·c in [128, 256)
          if (lane == 0 && (G >= 4 || warp < G)) {
            qs[h] = p.scale_log2 * __uint_as_float(static_cast<uint32_t>(127 - 7 + e) << 23);  // scale_log2 / c
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) x[i] *= c;
#pragma unroll
          for (int term = 0; term < t8::kTermsQ; ++term) {
            float d[4];
            const uint32_t word = t8::e4m3_pair(x[0], x[1], d[0], d[1]) | (t8::e4m3_pair(x[2], x[3], d[2], d[3]) << 16);
            const int n = term * G + h;
            const int col = 4 * lane;  // dims 4·lane .. +3 (byte offset within the 128-byte row)
            *reinterpret_cast<uint32_t*>(qbuf + (n >> 3) * 1024 + (n & 7) * 128 + ((((col >> 4) ^ (n & 7))) << 4) +
                                         (col & 15)) = word;
#pragma unroll
            for (int i = 0; i < 4; ++i) x[i] = (x[i] - d[i]) * 16.f;
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(L::kBQFull));
      // the per-head scales are read by every thread
      __syncwarp();
      fail = t8::softmax_bar_any(fail);
      if (fail) {
        t8::abort_softmax_impl(abort_flag);
        break;
      }
      float sw[G];
#pragma unroll
      for (int h = 0; h < G; ++h) sw[h] = qs[h];

      float m[G], l[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
      }
      for (int c = 0; c < nc; ++c, ++j) {
        const int a = u.t0 + c * t8::kTok;
        const int nv = min(t8::kTok, u.t1 - a);
        // ---- scores of token t ----
        const bool got = __all_sync(0xffffffffu, mbar_wait_sleep(bar(L::kBSFull + (j & 1)), (j >> 1) & 1, abort_flag));
        uint32_t sr[NS_] = {};
        if (got) {
          tc::fence_after_sync();
#pragma unroll
          for (int k = 0; k < NS_ / 8; ++k) tc::ld_32x32b_x8(tmem + lane_base + t8::kColS + (j & 1) * 32 + 8 * k, sr + 8 * k);
          tc::wait_ld();
        }
        tc::fence_before_sync();
        mbar_arrive(bar(L::kBSFree + (j & 1)));
        fail |= !got;
        float s[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float dot = __uint_as_float(sr[h]) + __uint_as_float(sr[G + h]) * 0.0625f +
                            __uint_as_float(sr[2 * G + h]) * 0.00390625f;
          s[h] = (t < nv && got) ? sw[h] * dot : -INFINITY;
        }
        {
          const float cm = t8::reduce_scatter<G, true>(s, lane);
          if (t8::scatter_first<G>(lane)) red[(j & 1) * 32 + warp * 8 + t8::scatter_head<G>(lane)] = cm;
        }
        __syncwarp();
        fail = t8::softmax_bar_any(fail);
        if (fail) {
          t8::abort_softmax_impl(abort_flag);
          break;
        }
        bool resc = false;
        float f[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float* rr = red + (j & 1) * 32 + h;
          const float mc = fmaxf(fmaxf(rr[0], rr[8]), fmaxf(rr[16], rr[24]));
          f[h] = 1.f;
          if (mc > m[h] + t8::kThreshold) {  // also when m is still -inf
            f[h] = m[h] == -INFINITY ? 0.f : fast_exp2(m[h] - mc);
            m[h] = mc;
            resc = resc || c > 0;
          }
        }
        if (resc) {
          // O^T holds chunks 0 .. c-1: once their last P·V is done, rescale it in place
          const bool okp = __all_sync(
              0xffffffffu, mbar_wait_sleep(bar(L::kBPFree + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag));
          fail |= !okp;
          if (okp) {
            tc::fence_after_sync();
            uint32_t o[NO];
#pragma unroll
            for (int k = 0; k < NO / 16; ++k) tc::ld_32x32b_x16(tmem + lane_base + t8::kColO + 16 * k, o + 16 * k);
            tc::wait_ld();
#pragma unroll
            for (int n = 0; n < t8::kTermsP * G; ++n) o[n] = __float_as_uint(__uint_as_float(o[n]) * f[n % G]);
#pragma unroll
            for (int k = 0; k < NO / 16; ++k) tc::st_32x32b_x16(tmem + lane_base + t8::kColO + 16 * k, o + 16 * k);
            tc::wait_st();
          }
#pragma unroll
          for (int h = 0; h < G; ++h) l[h] *= f[h];
        }

        // ---- P = 2^(s - m) as four e4m3 terms: byte i*G + h of token t's row ----
        const bool okf = __all_sync(
            0xffffffffu, mbar_wait_sleep(bar(L::kBPFree + (j & 1)), ((j >> 1) & 1) ^ 1, abort_flag));  // P·V of j-2
        fail |= !okf;
        float x[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          x[h] = fast_exp2(s[h] - m[h]);
          l[h] += x[h];
        }
        uint32_t pw[NO / 4];
#pragma unroll
        for (int i = 0; i < NO / 4; ++i) pw[i] = 0u;
#pragma unroll
        for (int term = 0; term < t8::kTermsP; ++term) {
          if constexpr (G == 1) {
            float d0, d1;
            const uint32_t c2 = t8::e4m3_pair(x[0], 0.f, d0, d1);
            pw[0] |= (c2 & 0xffu) << (8 * term);
            x[0] = (x[0] - d0) * 16.f;
          } else {
#pragma unroll
            for (int h = 0; h < G; h += 2) {
              float d0, d1;
              const uint32_t c2 = t8::e4m3_pair(x[h], x[h + 1], d0, d1);
              const int n = term * G + h;  // even: the pair fills half of a word
              pw[n >> 2] |= c2 << (8 * (n & 3));
              x[h] = (x[h] - d0) * 16.f;
              x[h + 1] = (x[h + 1] - d1) * 16.f;
            }
          }
        }
        unsigned char* pb = smem + L::kOffP + (j & 1) * L::kPBuf;
#pragma unroll
        for (int g16 = 0; g16 < NO / 16; ++g16) {
          *reinterpret_cast<uint4*>(pb + g16 * 2048 + t * 16) =
              make_uint4(pw[4 * g16], pw[4 * g16 + 1], pw[4 * g16 + 2], pw[4 * g16 + 3]);
        }
        if (nv < t8::kTok && t >= nv) {
          // V rows past the sequence end (stale codes may be NaN) become zeros;
          // the chunk's fill has landed (its K was read by the score MMAs)
          const int s = j % NSt;
          if (mbar_wait(bar(L::kBFull + s), (j / NSt) & 1, abort_flag)) {
            uint4* vrow = reinterpret_cast<uint4*>(smem + s * t8::kStageBytes + t8::kTileBytes + t * t8::kD);
#pragma unroll
            for (int i = 0; i < t8::kD / 16; ++i) vrow[i] = make_uint4(0u, 0u, 0u, 0u);
          } else {
            fail = true;
          }
        }
        fence_proxy_async_smem();
        tc::fence_before_sync();
        mbar_arrive(bar(L::kBPFull + (j & 1)));
      }
      if (fail) break;

      // ---- unit epilogue: row sums over the 128 threads, O^T out of tensor memory ----
      float* lsum = red + 64;  // [4 warps][8 heads], after the two chunk-max buffers
      {
        const float ls = t8::reduce_scatter<G, false>(l, lane);
        if (t8::scatter_first<G>(lane)) lsum[warp * 8 + t8::scatter_head<G>(lane)] = ls;
      }
      const bool okd =
          __all_sync(0xffffffffu, mbar_wait_sleep(bar(L::kBPFree + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag));
      fail |= !okd;
      __syncwarp();
      fail = t8::softmax_bar_any(fail);
      if (fail) {
        t8::abort_softmax_impl(abort_flag);
        break;
      }
      tc::fence_after_sync();
      uint32_t o[NO];
#pragma unroll
      for (int k = 0; k < NO / 16; ++k) tc::ld_32x32b_x16(tmem + lane_base + t8::kColO + 16 * k, o + 16 * k);
      tc::wait_ld();
      tc::fence_before_sync();
      const bool single = u.nparts == 1;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float lt = (lsum[h] + lsum[8 + h]) + (lsum[16 + h] + lsum[24 + h]);
        float num = 0.f;
#pragma unroll
        for (int term = t8::kTermsP - 1; term >= 0; --term) num = num * 0.0625f + __uint_as_float(o[term * G + h]);
        const int64_t row = row0 + h;
        if (single) {
          p.out[row * t8::kD + t] = lt > 0.f ? p.v_scale * num / lt : 0.f;
        } else {
          const int64_t pr = row * p.max_parts + u.part;
          p.part_o[pr * t8::kD + t] = p.v_scale * num;
          if (t == 0) {
            p.part_m[pr] = m[h];
            p.part_l[pr] = lt;
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == t8::kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, t8::kTmemCols);
  }
}

}  // namespace pkv
