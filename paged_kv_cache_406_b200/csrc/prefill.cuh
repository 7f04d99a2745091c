// Paged prefill attention on the fifth-generation tensor cores (tcgen05).
//
// What it computes (vLLM production page §2 and optimisation-overview page
// §2.3: chunked prefill): sequence b brings n_b new query rows (packed in q
// from q_start[b]); their K/V are already in the pool, which holds
// seq_lens[b] = L_b tokens.  Row i sits at position L_b - n_b + i and attends
// causally to tokens 0 .. that position through the block table (vLLM paging
// page §3 phase 2), KV head h / G, fp32 output.
//
// A tile is 256 rows = 256/G query tokens x the G query heads of one KV head,
// in two halves A and B of 128 rows (one M = 128 MMA tile each), so a GQA
// group turns into full MMA tiles even for short chunks; persistent CTAs (one
// per SM) take tiles one after another.  Keys come in chunks of 128 tokens
// (128/block_size physical blocks, one TMA box per block and head_dim half),
// each loaded once for both halves.  Per chunk j and half h:
//
//   S_h = Q_h · K_jᵀ      tcgen05.mma, 128x128x128, A and B from shared memory,
//                         fp32 in tensor memory
//   P_h = 2^(S_h·scale·log2e - m)   4 softmax warps per half, one row per
//                         thread, written back over S_h as bf16 hi + lo, or one
//                         f16
//   O_h += P_h · V_j      tcgen05.mma, A (P) from tensor memory, B (V) from
//                         shared memory
//
// The halves ping-pong: the MMA warp issues P·V of one half and q·Kᵀ of its
// next chunk as soon as that half's P is written, so the tensor core works on
// one half while the other half's softmax runs.  With a single 128-row tile,
// each chunk's P·V waited for the S -> softmax -> P round trip of the same
// tile, and the tensor core idled half of the time even with no softmax work
// at all; two halves also load K/V once per 256 rows.
//
// Warp roles (384 threads): warps 0-3 softmax of half A, 4-7 of half B
// (thread = row = TMEM lane of its warp's lane quarter, warp mod 4), warps 8
// and 9 TMA producers (K with Q, V), warp 10 MMA issuer (lane 0) and TMEM
// owner, warp 11 idle (it completes the fourth warpgroup, whose registers go
// to the softmax warpgroups).  Tensor memory (512 columns): S / P of half h
// at column 128 h (P hi in the first 64 columns, P lo in the next 64; a single
// f16 P in the first 64), O of half h at 256 + 128 h.
// Shared memory: Q of both halves 64 KB, K and V rings of 32 KB stages, and
// 4 KB per softmax warp through which its output rows leave in 128-byte
// pieces.  Keeping P in tensor memory spares shared memory 128 KB of traffic
// per chunk (P written and read back), which bounded the first version of
// this kernel.
//
// Pipeline per chunk j: P·V_A(j), q·Kᵀ_A(j+1), P·V_B(j), q·Kᵀ_B(j+1).  A half
// has one S / P buffer: q·Kᵀ of its next chunk overwrites P only after the
// P·V that reads it (the tensor core runs a thread's MMAs in order), and the
// commit of S_h(j) covers P·V_h(j-1), so a softmax warp that sees S_h(j) may
// rescale O_h at once.  The running max moves lazily (only by more than 8 in
// log2 units), as in the decode kernels.
//
// P precision: a single bf16 P (8 significant bits) misses the 2e-3 output
// tolerance at early positions (few keys of comparable weight), so for bf16
// pools P is stored as hi + lo halves (about 16 bits, within about 1e-5) at
// the cost of a second P·V pass (one MMA per half).  For f16 pools a single
// f16 P (11 bits: weights within 2^-11 relative, outputs within about 5e-4
// of the output scale) meets the tolerance, and P·V is one pass.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>

#include "device_common.cuh"
#include "tcgen05.cuh"

namespace pkv {

struct PrefillParams {
  const int32_t* block_tables;  // [num_seqs, max_blocks]
  const int32_t* seq_lens;      // [num_seqs] tokens in the pool, chunk included
  const int32_t* q_start;       // [num_seqs + 1] first q row of each sequence
  float* out;                   // [num_q_tokens, num_q_heads, 128]
  int32_t num_seqs, num_q_heads, num_kv_heads, num_blocks, max_blocks, block_size;
  int32_t num_q_tokens, max_q_len, n_tiles;
  float scale_log2;  // scale · log2(e), positive
  // bf16 pools with a staged f16 copy of V (v_staged != 0): P·V runs as one
  // f16 pass over the copy, unless the staging recorded a value beyond the
  // f16 range (*v_range == epoch), in which case it runs as the two bf16
  // passes (P hi and lo) over the pool's V (two launches, see the kernel)
  int32_t v_staged;
  uint32_t epoch;
  const uint32_t* v_range;
  // Test support for the bounded waits (pkv_debug_stall_prefill): the K
  // producer of CTA `stall_cta` skips its first K chunk, so the MMA warp's
  // wait for it runs out.  stall_cta < 0 in normal calls.
  int32_t stall_cta = -1;
};

#ifndef PKV_PREFILL_STAGES
#define PKV_PREFILL_STAGES 2
#endif

namespace pf {
constexpr int kRows = 128;              // MMA M: query rows per half tile
constexpr int kTileRows = 256;          // query rows per tile (halves A and B)
constexpr int kKeys = 128;              // keys per chunk (S columns, P·V contraction)
constexpr int kHeadDim = 128;
constexpr uint32_t kSlab = 128 * 128;   // 128 rows x 64 elements x 2 bytes
constexpr uint32_t kTile = 2 * kSlab;   // 128 rows x head_dim 128
constexpr int kStages = PKV_PREFILL_STAGES;  // K and V ring depth
constexpr int kSoftmaxThreads = 256;    // warps 0-7
constexpr int kProducerK = 8, kProducerV = 9, kMmaWarp = 10;
constexpr int kThreads = 384;  // warp 11 only completes the producer warpgroup
constexpr uint32_t kOffQ = 0;                              // Q of half h at h * kTile
constexpr uint32_t kOffK = kOffQ + 2 * kTile;
constexpr uint32_t kOffV = kOffK + kStages * kTile;
constexpr uint32_t kStageWarp = 32 * 32 * 4;               // a warp's 32 rows x 32 fp32 output columns
constexpr uint32_t kOffStage = kOffV + kStages * kTile;
constexpr uint32_t kOffBar = kOffStage + 8 * kStageWarp;
constexpr size_t kSmemBytes = kOffBar + 256 + 1024;  // barriers, flags; 1024 B alignment slack
static_assert(kSmemBytes <= 227 * 1024, "one CTA's shared memory (227 KB at most on sm_100)");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;   // S / P of half h at 128 h, O of half h at 256 + 128 h
constexpr float kRescale = 8.0f;
constexpr unsigned kAll = 0xffffffffu;
// mbarrier slots; Q, S, P, O-done and O-free come once per half
enum : int { kQFull = 0, kQEmpty = 2, kKFull = 4, kKEmpty = kKFull + kStages, kVFull = kKEmpty + kStages,
             kVEmpty = kVFull + kStages, kSFull = kVEmpty + kStages, kPFull = kSFull + 2, kODone = kPFull + 2,
             kOFree = kODone + 2, kTileReady = kOFree + 2, kTileFree = kTileReady + 2, kDrain = kTileFree + 2,
             kNumBars = kDrain + 1 };
static_assert(kNumBars * 8 + 16 <= 256, "barriers, flags and tile slots fit the reserved 256 bytes");
// arrivals per phase: P-full and O-free by lane 0 of each of a half's four
// softmax warps, once the whole warp's tensor-memory accesses are done;
// tile-free by lane 0 of the V producer, the MMA warp and the eight softmax
// warps
__host__ __device__ constexpr uint32_t bar_count(int i) {
  return (i >= kPFull && i < kPFull + 2) || (i >= kOFree && i < kOFree + 2) ? 4u
         : (i >= kTileFree && i < kTileFree + 2)                            ? 10u
                                                                            : 1u;
}
// S-full and P-full of a half complete once per chunk and O-done / O-free
// once per tile; a half's next phase needs the MMA warp or the softmax warps
// of that half to have moved on, so no waiter can ever be a whole phase behind
}  // namespace pf

__device__ __forceinline__ void tma_load_3d_nohint(uint32_t dst, const void* tmap, int32_t x, int32_t y, int32_t z,
                                                   uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* tmap, int32_t x, int32_t y, int32_t z, int32_t w,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
      : "memory");
}

// P as two 16-bit halves, packed in pairs (x0 in the low half): hi + lo
// carries about 16 significant bits.  bf16: hi is the truncated top half of
// the fp32 value (a byte permute), lo the rounded remainder (exact in fp32).
template <typename T>
__device__ __forceinline__ void split_hi_lo(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  split_pack<T>(x0, x1, hi, lo);
}

template <>
__device__ __forceinline__ void split_hi_lo<__nv_bfloat16>(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  // hi: the top 16 bits of each fp32 value; lo: the top 16 bits of the
  // (exact) remainder.  Both truncations are byte permutes on the integer
  // pipe, which keeps the special-function pipe (busy with the
  // exponentials) free of conversions; hi + lo is within 2^-16 of x.
  const uint32_t u0 = __float_as_uint(x0), u1 = __float_as_uint(x1);
  hi = __byte_perm(u0, u1, 0x7632);
  // x - trunc(x), both lanes in one packed FMA (exact: the remainder fits)
  const float2 r = __ffma2_rn(make_float2(__uint_as_float(u0 & 0xffff0000u), __uint_as_float(u1 & 0xffff0000u)),
                              make_float2(-1.f, -1.f), make_float2(x0, x1));
  lo = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x7632);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// ---------------------------------------------------------------------------
// V staged as f16 for bf16 pools (one pass per call, before the prefill
// kernel).  bf16 carries 8 significant bits and f16 11, so every bf16 value
// of magnitude in [2^-14, 65504] converts exactly; smaller ones round to f16
// subnormals (absolute error at most 2^-25).  A finite value above 65504 has
// no f16 counterpart: the kernel then writes the call's epoch into *range and
// the prefill kernel keeps the bf16 hi + lo path over the pool's own V.
// Layout of the copy: [num_seqs][max_blocks][Hkv][block_size][128] f16; the
// blocks of sequence b past ceil(seq_lens[b] / block_size) are not written.
// Grid: y strides over the sequences, x over the blocks of one; a CTA copies
// whole blocks (one table read each), four 16-byte pieces per thread in
// flight.
// ---------------------------------------------------------------------------
struct VStageArgs {
  const int32_t* block_tables;
  const int32_t* seq_lens;
  const uint4* v_pool;  // bf16 pool, 16 bytes = 8 elements
  uint4* staged;        // f16 copy
  uint32_t* range;
  uint32_t epoch;
  int32_t num_seqs, num_blocks, max_blocks, block_size, block_pieces;  // pieces: Hkv * block_size * 128 / 8
};

// Eight bf16 values (16 bytes) to eight f16 values; `over` is set if a finite
// value lies beyond the f16 range.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 w, bool& over) {
  const uint32_t in[4] = {w.x, w.y, w.z, w.w};
  uint32_t res[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // bf16 is the top half of an fp32: widening is a shift
    const float lo = __uint_as_float(in[k] << 16), hi = __uint_as_float(in[k] & 0xffff0000u);
    over |= (fabsf(lo) > 65504.f && fabsf(lo) != INFINITY) || (fabsf(hi) > 65504.f && fabsf(hi) != INFINITY);
    const __half2 h = __floats2half2_rn(lo, hi);
    res[k] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(res[0], res[1], res[2], res[3]);
}

__global__ void __launch_bounds__(256) stage_v_f16_kernel(const VStageArgs a) {
  // launched programmatically serialised: the previous kernel of the stream
  // (the append of the chunk's rows) is complete before anything is read
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int kUnroll = 4;
  bool over = false;
  const int pieces = a.block_pieces;
  for (int b = blockIdx.y; b < a.num_seqs; b += gridDim.y) {
    int L = a.seq_lens[b];
    L = L < 0 ? 0 : min(L, a.max_blocks * a.block_size);
    const int nblk = (L + a.block_size - 1) / a.block_size;
    const int32_t* trow = a.block_tables + static_cast<int64_t>(b) * a.max_blocks;
    for (int j = blockIdx.x; j < nblk; j += gridDim.x) {
      int phys = trow[j];
      if (static_cast<unsigned>(phys) >= static_cast<unsigned>(a.num_blocks)) {
        if (threadIdx.x == 0) record_error(PKV_ERR_BAD_BLOCK);
        phys = 0;
      }
      const uint4* src = a.v_pool + static_cast<int64_t>(phys) * pieces;
      uint4* dst = a.staged + (static_cast<int64_t>(b) * a.max_blocks + j) * pieces;
      int i = threadIdx.x;
      for (; i + (kUnroll - 1) * 256 < pieces; i += kUnroll * 256) {
        uint4 w[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) w[u] = src[i + u * 256];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) dst[i + u * 256] = bf16x8_to_f16x8(w[u], over);
      }
      for (; i < pieces; i += 256) dst[i] = bf16x8_to_f16x8(src[i], over);
    }
  }
  if (__any_sync(0xffffffffu, over) && (threadIdx.x & 31) == 0) atomicExch(a.range, a.epoch);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the prefill instances wait for this grid
}

// kF16P: one f16 P and one P·V pass over f16 V (the pool's own for f16 pools,
// the staged copy for bf16 pools); otherwise (bf16 only) P as bf16 hi + lo
// halves, two passes over the pool's bf16 V.  A bf16 call with staged V
// launches both instances: each reads the staging record first and the one
// whose case does not hold returns at once (the record says whether some V
// value lay beyond the f16 range), so each instance carries one P path only.
template <typename T, int G, bool kF16P>
__global__ void __launch_bounds__(pf::kThreads, 1)
    prefill_tc_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                      unsigned int* __restrict__ tile_ctr) {
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  constexpr int QT = pf::kRows / G;  // query tokens per half tile
  constexpr int QT2 = 2 * QT;        // query tokens per tile
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  static_assert(kBf16 || kF16P, "f16 pools take the one-pass f16 P");
  constexpr bool f16p = kF16P;
  // Launched programmatically serialised (behind the V staging, or the other
  // instance of a staged bf16 call, or whatever the stream ran before): the
  // next instance may be scheduled at once, and this one waits for the
  // previous kernel (so for the staging and the append before it) before
  // reading anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (kBf16 && p.v_staged) {
    const bool beyond = *p.v_range == p.epoch;
    if (beyond == kF16P) return;  // the other instance of this call does the work
  }
  constexpr bool v_from_stage = kBf16 && kF16P;  // tmap_v then maps the staged f16 copy

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t base = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + pf::kOffBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + pf::kNumBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + pf::kNumBars) + 1;
  volatile int* tile_slot = reinterpret_cast<volatile int*>(bars + pf::kNumBars) + 2;  // two slots
  auto bar = [&](int i) { return smem_addr(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < pf::kNumBars; ++i) mbar_init(bar(i), pf::bar_count(i));
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == pf::kMmaWarp) {
    tc::tmem_alloc(smem_addr(tmem_slot), pf::kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == pf::kProducerK && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int total = p.n_tiles * p.num_seqs * p.num_kv_heads;

  // Persistent CTAs (one per SM).  The K producer draws tile numbers from a
  // counter and publishes each in one of two slots (tile-ready barrier); the
  // other roles read it and hand the slot back (tile-free barrier).  Tile t
  // is the (sequence b, KV head g, tile of QT2 query tokens) of the order:
  // sequence by sequence, and within a sequence tile by tile, most keys
  // first, each tile for all KV heads.  The tiles in flight at any time then
  // share a few sequences' K/V in L2 (taking one tile index of every
  // sequence together re-read K/V from DRAM about 7x), and each sequence
  // hands out its short tiles last (taking all tiles of one KV head before
  // the next left the longest tiles of the last sequence's last heads to
  // the end of the launch, with most SMs idle); drawing them from a counter
  // balances the SMs as they finish.  Each role moves on
  // to the next tile as soon as its own part is done, so the next tile's Q
  // and K loads and its first q·Kᵀ run during this tile's last P·V and
  // output; only a half's first P·V of the next tile waits for its output to
  // have left tensor memory (O-free), and its next Q load for its last q·Kᵀ
  // (Q-empty).
  // The barriers count phases across tiles: gc is the number of key chunks
  // and tv the number of tiles a role has done before the current one (the
  // same sequence in every role); chunk j of a tile is chunk gc + j.
  struct Tile {
    int b, g, q0, n, L, tok0, ctx, pos_min, nc, nblk;
    bool valid;
  };
  auto tile_of = [&](int t) {
    Tile d{};
    const int per_seq = p.n_tiles * p.num_kv_heads;
    d.b = t / per_seq;
    const int w = t - d.b * per_seq;
    const int tile = p.n_tiles - 1 - w / p.num_kv_heads;  // most keys first
    d.g = w % p.num_kv_heads;
    d.q0 = p.q_start[d.b];
    const int q1 = p.q_start[d.b + 1];
    d.n = q1 - d.q0;
    d.L = p.seq_lens[d.b];
    d.tok0 = tile * QT2;  // chunk-relative first token of the tile
    const bool args_ok = !(d.n < 0 || d.q0 < 0 || q1 > p.num_q_tokens || d.n > d.L || d.n > p.max_q_len ||
                           d.L > p.max_blocks * p.block_size);
    if (!args_ok && tile == 0 && warp == pf::kProducerK && lane == 0) record_error(PKV_ERR_INVALID_ARG);
    d.valid = args_ok && d.tok0 < d.n;
    if (!d.valid) return d;
    d.ctx = d.L - d.n;
    d.pos_min = d.ctx + d.tok0;
    const int pos_max = min(d.L - 1, d.ctx + d.tok0 + QT2 - 1);
    d.nc = pos_max / pf::kKeys + 1;  // key chunks this tile attends to
    d.nblk = (d.L + p.block_size - 1) / p.block_size;
    return d;
  };
  // the tile number of round ti, for every role but the K producer (which
  // publishes it): returns total when there are no more tiles (or on abort)
  auto read_tile = [&](int ti) -> int {
    int t = total;
    if (lane == 0) {
      if (mbar_wait_sleep(bar(pf::kTileReady + (ti & 1)), (ti >> 1) & 1, abort_flag)) t = tile_slot[ti & 1];
      mbar_arrive(bar(pf::kTileFree + (ti & 1)));
    }
    return __shfl_sync(pf::kAll, t, 0);
  };
  const int BS = p.block_size;
  int issued = 0, q_issued[2] = {0, 0};  // producers: fills issued (chunks, Q tiles of each half) in the CTA's count
  int skipped = -1;                       // the K producer's chunk left out by the stall test support

  // Registers: the kernel is launched at 168 a thread (384 x 168 = 64512);
  // the producer / MMA warpgroup (warps 8-11) drops to 112 and the two softmax
  // warpgroups rise to 184 (128 x 112 + 256 x 184 = 61440, within the launch's
  // total, so the increase never waits for long): the softmax rows (128
  // scores a thread) then fit in registers without spilling.
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 112;\n" ::: "memory");
    if (warp == pf::kProducerK || warp == pf::kProducerV) {
      // ----------------------------- TMA producers -----------------------------
      // One warp streams K chunks (and Q), the other V chunks, each through its
      // own ring: K runs ahead of V (q·Kᵀ of chunk j+1 is issued right after
      // each half's P·V of chunk j, while V's stages free only as both halves'
      // P·V complete; a single producer alternating K and V held K behind V's
      // refills).
      const int kv = warp == pf::kProducerV ? 1 : 0;
      bool ok = true;
      int gc = 0, tv = 0;
      for (int ti = 0; ok; ++ti) {
        int t;
        if (kv == 0) {
          t = total;
          if (lane == 0) {
            // the slot's previous tile has been read by every other role
            const bool free = ti < 2 || mbar_wait_sleep(bar(pf::kTileFree + (ti & 1)), ((ti >> 1) - 1) & 1, abort_flag);
            if (!free && !*abort_flag) {
              record_error(PKV_ERR_DEVICE_TIMEOUT);
              *abort_flag = 1;
            }
            const unsigned ticket = (!free || *abort_flag) ? static_cast<unsigned>(total) : atomicAdd(tile_ctr, 1u);
            t = ticket >= static_cast<unsigned>(total) ? total : static_cast<int>(ticket);
            tile_slot[ti & 1] = t;
            mbar_arrive(bar(pf::kTileReady + (ti & 1)));
          }
          t = __shfl_sync(pf::kAll, t, 0);
        } else {
          t = read_tile(ti);
        }
        if (t >= total) break;
        const Tile d = tile_of(t);
        if (!d.valid) continue;
        const int b = d.b, g = d.g, nc = d.nc, nblk = d.nblk;
        if (kv == 0) {
          // Q of a half of the previous tile is no longer read once that half's
          // last q·Kᵀ is done; half h holds tokens tok0 + h * QT .. + QT - 1
          // (rows token * G + head; tokens past q's end read as zeros)
          for (int h = 0; h < 2 && ok; ++h) {
            if (tv > 0) ok = __all_sync(pf::kAll, mbar_wait_sleep(bar(pf::kQEmpty + h), (tv - 1) & 1, abort_flag));
            if (!ok) break;
            if (lane == 0) {
              const uint32_t dst = base + pf::kOffQ + h * pf::kTile;
              mbar_arrive_expect_tx(bar(pf::kQFull + h), pf::kTile);
              tma_load_4d(dst, &tmap_q, 0, 0, g * G, d.q0 + d.tok0 + h * QT, bar(pf::kQFull + h));
              tma_load_4d(dst + pf::kSlab, &tmap_q, 0, 1, g * G, d.q0 + d.tok0 + h * QT, bar(pf::kQFull + h));
            }
            q_issued[h] = tv + 1;
          }
          if (!ok) break;
        }
        const int32_t* trow = p.block_tables + static_cast<int64_t>(b) * p.max_blocks;
        const int nbc = pf::kKeys / BS;                              // blocks per chunk
        const uint32_t box_bytes = static_cast<uint32_t>(BS) * 128;  // one block, one head_dim half
        const uint32_t full0 = bar(kv ? pf::kVFull : pf::kKFull), empty0 = bar(kv ? pf::kVEmpty : pf::kKEmpty);
        // V from the staged f16 copy: block j of sequence b sits at b * max_blocks + j, no table lookup
        const bool staged = kv && v_from_stage;
        const void* map = kv ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k);
        const uint32_t ring = base + (kv ? pf::kOffV : pf::kOffK);
        for (int j = 0; j < nc && ok; ++j) {
          const int s = (gc + j) % pf::kStages;
          const uint32_t ph = (((gc + j) / pf::kStages) & 1) ^ 1;
          const int jb = j * nbc;
          const int nload = min(nbc, nblk - jb);  // blocks past the sequence end are not read
          int phys = 0;
          if (lane < nload) {
            if (staged) {
              phys = b * p.max_blocks + jb + lane;
            } else {
              phys = trow[jb + lane];
              if (static_cast<unsigned>(phys) >= static_cast<unsigned>(p.num_blocks)) {
                record_error(PKV_ERR_BAD_BLOCK);
                phys = 0;
              }
            }
          }
          const int32_t y = (phys * p.num_kv_heads + g) * BS;
          const uint32_t full = full0 + 8 * s;
          ok = __all_sync(pf::kAll, mbar_wait_sleep(empty0 + 8 * s, ph, abort_flag));
          if (!ok) break;
          if (kv == 0 && gc + j == 0 && p.stall_cta == static_cast<int>(blockIdx.x)) {
            skipped = 0;  // test support: the CTA's first K chunk never arrives
          } else {
            if (lane == 0) mbar_arrive_expect_tx(full, static_cast<uint32_t>(nload) * 2u * box_bytes);
            __syncwarp();
            if (lane < nload) {
              const uint32_t dst = ring + s * pf::kTile + lane * box_bytes;
              tma_load_3d_nohint(dst, map, 0, y, 0, full);
              tma_load_3d_nohint(dst + pf::kSlab, map, 0, y, 1, full);
            }
          }
          issued = gc + j + 1;
        }
        gc += nc;
        ++tv;
      }
      if (!ok && lane == 0) {
        record_error(PKV_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
      }
      // no copy may still be landing when the CTA exits (a timeout can leave
      // fills unconsumed): wait (bounded) for the last fill of each stage and Q
      if (lane == 0) {
        const uint32_t full0 = bar(kv ? pf::kVFull : pf::kKFull);
        if (kv == 0)
          for (int h = 0; h < 2; ++h)
            if (q_issued[h] > 0) mbar_drain(bar(pf::kQFull + h), (q_issued[h] - 1) & 1);
        for (int s = 0; s < pf::kStages && s < issued; ++s) {
          const int last = s + (issued - 1 - s) / pf::kStages * pf::kStages;  // last chunk that used stage s
          if (last != skipped) mbar_drain(full0 + 8 * s, (last / pf::kStages) & 1);  // a skipped fill never lands
        }
      }
      __syncwarp();
    } else if (warp == pf::kMmaWarp) {
      // ------------------------------- MMA issuer -------------------------------
      const uint32_t id_s = tc::idesc_f16(kBf16, false, pf::kRows, pf::kKeys);
      // P·V: f16 P and f16 V in one pass, or bf16 P hi and lo over bf16 V
      const uint32_t id_o = tc::idesc_f16(kBf16 && !f16p, true, pf::kRows, pf::kHeadDim);
      constexpr int parts = f16p ? 1 : 2;
      bool ok = true;
      int gc = 0, tv = 0;
      for (int ti = 0; ok; ++ti) {
        const int t = read_tile(ti);
        if (t >= total) break;
        const Tile d = tile_of(t);
        if (!d.valid) continue;
        const int nc = d.nc;
        if (lane == 0) {
          // S_h = Q_h · K_jᵀ into half h's S / P columns; the K stage has landed
          auto issue_s = [&](int h, int j) {
            const uint32_t kst = base + pf::kOffK + ((gc + j) % pf::kStages) * pf::kTile;
            const uint32_t qh = base + pf::kOffQ + h * pf::kTile;
  #pragma unroll
            for (int kk = 0; kk < pf::kHeadDim / 16; ++kk) {
              const uint32_t off = (kk >> 2) * pf::kSlab + (kk & 3) * 32;
              tc::mma_f16_ss(tmem + pf::kColS + h * pf::kKeys, tc::sw128_desc(qh + off, 16, 1024),
                             tc::sw128_desc(kst + off, 16, 1024), id_s, kk > 0 ? 1u : 0u);
            }
            tc::commit(bar(pf::kSFull + h));
          };
          // O_h += P_h · V_j (P hi in the first 64 columns of the half's buffer, P lo in the next 64)
          auto issue_pv = [&](int h, int j) {
            const uint32_t vst = base + pf::kOffV + ((gc + j) % pf::kStages) * pf::kTile;
            const uint32_t pt = tmem + pf::kColS + h * pf::kKeys;
  #pragma unroll
            for (int part = 0; part < parts; ++part) {
  #pragma unroll
              for (int kk = 0; kk < pf::kKeys / 16; ++kk) {
                const uint32_t bv = vst + kk * 16 * 128;  // 16 keys of 128-byte rows
                tc::mma_f16_ts(tmem + pf::kColO + h * pf::kHeadDim, pt + part * (pf::kKeys / 2) + kk * 8,
                               tc::sw128_desc(bv, pf::kSlab, 1024), id_o, (j > 0 || part > 0 || kk > 0) ? 1u : 0u);
              }
            }
          };
          auto wait_k = [&](int j) {
            const int gj = gc + j;
            const bool r = mbar_wait_sleep(bar(pf::kKFull + gj % pf::kStages), (gj / pf::kStages) & 1, abort_flag);
            tc::fence_after_sync();
            return r;
          };
          // the tile's first q·Kᵀ of both halves
          ok = mbar_wait_sleep(bar(pf::kQFull), tv & 1, abort_flag) &&
               mbar_wait_sleep(bar(pf::kQFull + 1), tv & 1, abort_flag) && wait_k(0);
          if (ok) {
            issue_s(0, 0);
            if (nc == 1) tc::commit(bar(pf::kQEmpty));  // half A's last q·Kᵀ
            issue_s(1, 0);
            if (nc == 1) tc::commit(bar(pf::kQEmpty + 1));
            tc::commit(bar(pf::kKEmpty + gc % pf::kStages));
          }
          for (int j = 0; j < nc && ok; ++j) {
            const int gj = gc + j;
            const int s = gj % pf::kStages;
            ok = mbar_wait_sleep(bar(pf::kVFull + s), (gj / pf::kStages) & 1, abort_flag);
            // half A: its P·V (after the previous tile's O_A has left tensor
            // memory), then its next q·Kᵀ, which waits for the next K stage
            if (ok && j == 0 && tv > 0) ok = mbar_wait_sleep(bar(pf::kOFree), (tv - 1) & 1, abort_flag);
            if (ok) ok = mbar_wait_sleep(bar(pf::kPFull), gj & 1, abort_flag);
            if (!ok) break;
            tc::fence_after_sync();
            issue_pv(0, j);
            if (j + 1 < nc) {
              if (!(ok = wait_k(j + 1))) break;
              issue_s(0, j + 1);
              if (j + 1 == nc - 1) tc::commit(bar(pf::kQEmpty));
            } else {
              tc::commit(bar(pf::kODone));  // O_A is complete once its last P·V is
            }
            // half B likewise; V_j and K_{j+1} are then free
            if (j == 0 && tv > 0) ok = mbar_wait_sleep(bar(pf::kOFree + 1), (tv - 1) & 1, abort_flag);
            if (ok) ok = mbar_wait_sleep(bar(pf::kPFull + 1), gj & 1, abort_flag);
            if (!ok) break;
            tc::fence_after_sync();
            issue_pv(1, j);
            tc::commit(bar(pf::kVEmpty + s));
            if (j + 1 < nc) {
              issue_s(1, j + 1);
              tc::commit(bar(pf::kKEmpty + (gj + 1) % pf::kStages));
              if (j + 1 == nc - 1) tc::commit(bar(pf::kQEmpty + 1));
            } else {
              tc::commit(bar(pf::kODone + 1));
            }
          }
        }
        ok = __shfl_sync(pf::kAll, ok, 0);
        gc += nc;
        ++tv;
      }
      if (lane == 0) {
        if (!ok) {
          record_error(PKV_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
        }
        // every MMA issued completes before tensor memory is freed
        tc::commit(bar(pf::kDrain));
        mbar_drain(bar(pf::kDrain), 0);
      }
      __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 184;\n" ::: "memory");
    // ------------------------------ softmax warps ------------------------------
    const int hh = warp >> 2;               // half of the tile
    const int r = (warp & 3) * 32 + lane;   // row of the half and TMEM lane
    const int R = hh * pf::kRows + r;       // row of the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t ts = trow + pf::kColS + hh * pf::kKeys;     // this half's S / P
    const uint32_t to = trow + pf::kColO + hh * pf::kHeadDim;  // this half's O
    unsigned char* vzero = smem + pf::kOffV;
    float4* wstage = reinterpret_cast<float4*>(smem + pf::kOffStage + warp * pf::kStageWarp);
    const float sl = p.scale_log2;
    bool ok = true;
    int gc = 0, tv = 0;
    for (int ti = 0; ok; ++ti) {
      const int t = read_tile(ti);
      if (t >= total) break;
      const Tile d = tile_of(t);
      if (!d.valid) continue;
      const int nc = d.nc, L = d.L, n = d.n, tok0 = d.tok0, pos_min = d.pos_min;
      const int tok = tok0 + R / G;
      const int pos = min(d.ctx + tok, L - 1);  // rows past the chunk end compute a copy of the last row
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < nc && ok; ++j) {
        const int gj = gc + j;           // chunk of the CTA
        const int s = gj % pf::kStages;  // K / V stage
        ok = __all_sync(pf::kAll, mbar_wait_sleep(bar(pf::kSFull + hh), gj & 1, abort_flag));
        if (!ok) break;
        tc::fence_after_sync();
        float x[pf::kKeys];  // raw scores q·k of this row's 128 keys
        {
          uint32_t raw[4][32];
#pragma unroll
          for (int q = 0; q < 4; ++q) tc::ld_32x32b_x32(ts + 32 * q, raw[q]);
          tc::wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < 32; ++i) x[32 * q + i] = __uint_as_float(raw[q][i]);
        }
        const int key0 = j * pf::kKeys;
        if (key0 + pf::kKeys - 1 > pos_min) {  // the diagonal: keys after a row's position are hidden
#pragma unroll
          for (int c = 0; c < pf::kKeys; ++c) x[c] = key0 + c <= pos ? x[c] : -INFINITY;
        }
        // row max with three-input maxima in four independent chains; the
        // scale is positive, so the max of the scaled scores is the scaled max
        float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int c = 4; c + 8 <= pf::kKeys; c += 8) {
          mx[0] = max3f(mx[0], x[c], x[c + 1]);
          mx[1] = max3f(mx[1], x[c + 2], x[c + 3]);
          mx[2] = max3f(mx[2], x[c + 4], x[c + 5]);
          mx[3] = max3f(mx[3], x[c + 6], x[c + 7]);
        }
        mx[0] = max3f(mx[0], x[pf::kKeys - 4], x[pf::kKeys - 3]);
        mx[1] = max3f(mx[1], x[pf::kKeys - 2], x[pf::kKeys - 1]);
        const float mc = fmaxf(max3f(mx[0], mx[1], mx[2]), mx[3]) * sl;
        float factor = 1.f;
        bool resc = false;
        if (j == 0) {
          m_used = mc;  // key 0 is visible to every row: finite
        } else if (mc > m_used + pf::kRescale) {
          factor = fast_exp2(m_used - mc);
          m_used = mc;
          resc = true;
        }
        // exponentials (arguments and sums two lanes at a time, packed f32x2),
        // each quarter of the row written as P hi and lo over S in tensor
        // memory as soon as it is done (the stores complete while the next
        // quarter is computed): key pair (2c, 2c+1) in column c (hi) and
        // 64 + c (lo)
        float2 sm[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(-m_used, -m_used);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
#pragma unroll
          for (int c = 32 * h; c < 32 * h + 32; c += 2) {
            const float2 a = __ffma2_rn(make_float2(x[c], x[c + 1]), sl2, nm2);  // hidden keys: -inf -> 0
            x[c] = fast_exp2(a.x);
            x[c + 1] = fast_exp2(a.y);
            sm[(c >> 1) & 3] = __fadd2_rn(sm[(c >> 1) & 3], make_float2(x[c], x[c + 1]));
          }
          if constexpr (!f16p) {
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) split_hi_lo<T>(x[32 * h + 2 * c], x[32 * h + 2 * c + 1], hi[c], lo[c]);
            tc::st_32x32b_x16(ts + 16 * h, hi);
            tc::st_32x32b_x16(ts + pf::kKeys / 2 + 16 * h, lo);
          } else {
            uint32_t ph[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const __half2 v = __floats2half2_rn(x[32 * h + 2 * c], x[32 * h + 2 * c + 1]);
              ph[c] = *reinterpret_cast<const uint32_t*>(&v);
            }
            tc::st_32x32b_x16(ts + 16 * h, ph);
          }
        }
        const float2 s01 = __fadd2_rn(sm[0], sm[1]), s23 = __fadd2_rn(sm[2], sm[3]);
        const float2 st = __fadd2_rn(s01, s23);
        l = l * factor + (st.x + st.y);

        if (__any_sync(pf::kAll, resc)) {
          // O still holds the sum up to chunk j-1: the commit of S(j), seen
          // above, covers P·V(j-1), which the MMA warp issued before it
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t o[32];
            tc::ld_32x32b_x32(to + 32 * q, o);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
            tc::st_32x32b_x32(to + 32 * q, o);
          }
        }
        if (hh == 0 && key0 + pf::kKeys > L) {
          // V rows past the sequence end hold stale or unwritten bytes: half
          // A zeroes them (before its P-full, so before either half's P·V
          // reads them) so that P = 0 there cannot meet a NaN pattern
          ok = __all_sync(pf::kAll, mbar_wait_sleep(bar(pf::kVFull + s), (gj / pf::kStages) & 1, abort_flag));
          if (!ok) break;
          const int v0 = L - key0;
          unsigned char* vst = vzero + s * pf::kTile;
          for (int idx = r; idx < (pf::kKeys - v0) * 16; idx += 128) {
            const int row = v0 + (idx >> 4), piece = idx & 15;
            *reinterpret_cast<uint4*>(vst + (piece >> 3) * pf::kSlab + row * 128 + (piece & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();  // zeroed V rows visible to the tensor core
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(pf::kPFull + hh));
      }
      // the MMA warp commits O-done after the half's last P·V
      if (ok) ok = __all_sync(pf::kAll, mbar_wait_sleep(bar(pf::kODone + hh), tv & 1, abort_flag));
      if (!ok) break;
      tc::fence_after_sync();
      // O goes out 32 columns at a time through this warp's 4 KB of shared
      // memory: each thread parks 128 bytes of its row, then each store
      // instruction writes 4 rows' 128-byte pieces, instead of 32 rows' 16
      // bytes straight from the tensor-memory layout.  The 16-byte piece c of
      // parked row k sits at slot c ^ (k mod 8), so the parking and the
      // row-wise reads are both free of bank conflicts.  Once the last
      // columns are loaded, O may be overwritten by the next tile's P·V.
      const float inv = 1.f / l;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tc::ld_32x32b_x32(to + 32 * q, o);
        tc::wait_ld();
        if (q == 3) {
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(pf::kOFree + hh));
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          wstage[lane * 8 + (i ^ (lane & 7))] =
              make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                          __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int kr = 4 * k + (lane >> 3), piece = lane & 7;  // parked row and its 16-byte piece
          const int rr = hh * pf::kRows + (warp & 3) * 32 + kr;    // row of the tile
          const int tk = tok0 + rr / G;
          if (tk < n) {  // rows past the chunk end are not written
            float4* orow = reinterpret_cast<float4*>(
                p.out + (static_cast<int64_t>(d.q0 + tk) * p.num_q_heads + d.g * G + rr % G) * pf::kHeadDim);
            orow[8 * q + piece] = wstage[kr * 8 + (piece ^ (kr & 7))];
          }
        }
        __syncwarp();  // the pieces are out before the next columns are parked
      }
      gc += nc;
      ++tv;
    }
    if (!ok && lane == 0) {
      record_error(PKV_ERR_DEVICE_TIMEOUT);
      *abort_flag = 1;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == pf::kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, pf::kTmemCols);
  }
  if (threadIdx.x == 0) {
    // the last CTA to finish re-arms the counter for the next launch that
    // uses this slot: every CTA has drawn its last ticket before it counts
    // itself done
    __threadfence();
    if (atomicAdd(tile_ctr + 1, 1u) == gridDim.x - 1) {
      atomicExch(tile_ctr, 0u);
      atomicExch(tile_ctr + 1, 0u);
    }
  }
}

}  // namespace pkv
