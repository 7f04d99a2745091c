// KV append kernels (plain 16-byte row copies and e4m3 quantisation), the
// block copy of copy-on-write, and the launch that appends a decode step's
// rows while it plans the decode.
#pragma once

#include <cuda_fp8.h>

#include <type_traits>

#include "decode.cuh"
#include "device_common.cuh"

namespace pkv {

// ---------------------------------------------------------------------------
// KV append: one thread per 16-byte chunk of one (token, kv head) row, K and V.
// vLLM paging page §3 phase 1: the new token is written into its slot.
// ---------------------------------------------------------------------------
// Token i's row goes into pool c for tok0[c] <= i < tok0[c + 1] (one pool
// unless a step spans pools of several block sizes); its slot is pool-local.
struct AppendArgs {
  const void* k_new;
  const void* v_new;
  const int32_t* slots;
  int64_t n_units;  // 16-byte chunks (copy) or 8-element groups (e4m3) over all (token, head) rows
  void* k_pool[kMaxPools];
  void* v_pool[kMaxPools];
  int32_t num_blocks[kMaxPools], block_size[kMaxPools], tok0[kMaxPools];
  int32_t n_pools, num_kv_heads, row_units;
  float k_inv, v_inv;  // e4m3 only: 1 / scale
};

// The pool of token `tok` and its destination fields.
struct AppendDst {
  unsigned char* k_pool;
  unsigned char* v_pool;
  int32_t num_blocks, block_size;
};

__device__ __forceinline__ AppendDst append_dst(const AppendArgs& a, int64_t tok) {
  int c = 0;
  if (a.n_pools > 1) c = (tok >= a.tok0[1] ? 1 : 0) + (a.n_pools > 2 && tok >= a.tok0[2] ? 1 : 0);
  return AppendDst{static_cast<unsigned char*>(pick3(a.k_pool, c)), static_cast<unsigned char*>(pick3(a.v_pool, c)),
                   pick3(a.num_blocks, c), pick3(a.block_size, c)};
}

__device__ __forceinline__ void append_chunk(const AppendArgs& a, int64_t i) {
  const uint4* __restrict__ k_new = static_cast<const uint4*>(a.k_new);
  const uint4* __restrict__ v_new = static_cast<const uint4*>(a.v_new);
  const int32_t row_chunks = a.row_units, num_kv_heads = a.num_kv_heads;
  const int32_t chunk = static_cast<int32_t>(i % row_chunks);
  const int64_t row = i / row_chunks;  // token * num_kv_heads + head
  const int32_t h = static_cast<int32_t>(row % num_kv_heads);
  const int64_t tok = row / num_kv_heads;
  const int32_t slot = a.slots[tok];
  if (slot < 0) return;  // padding token
  const AppendDst t = append_dst(a, tok);
  uint4* __restrict__ k_pool = reinterpret_cast<uint4*>(t.k_pool);
  uint4* __restrict__ v_pool = reinterpret_cast<uint4*>(t.v_pool);
  const int32_t block_size = t.block_size;
  const int32_t blk = slot / block_size, off = slot - blk * block_size;
  if (blk >= t.num_blocks) {
    if (chunk == 0 && h == 0) record_error(PKV_ERR_BAD_BLOCK);
    return;
  }
  const int64_t dst = ((static_cast<int64_t>(blk) * num_kv_heads + h) * block_size + off) * row_chunks + chunk;
  k_pool[dst] = k_new[i];
  v_pool[dst] = v_new[i];
}

__global__ void __launch_bounds__(256) kv_append_kernel(const AppendArgs a) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < a.n_units) append_chunk(a, i);
  // a programmatically serialised successor (the prefill's V staging) may be
  // scheduled now; it still waits for this grid's writes before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Block copy for copy-on-write (vLLM paging page §3 phase 3): pair y copies
// one whole block of K and of V, every head and offset.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                                          const int32_t* __restrict__ pairs, int32_t num_blocks,
                                                          int64_t block_chunks) {
  const int32_t src = pairs[2 * blockIdx.y], dst = pairs[2 * blockIdx.y + 1];
  if (static_cast<unsigned>(src) >= static_cast<unsigned>(num_blocks) ||
      static_cast<unsigned>(dst) >= static_cast<unsigned>(num_blocks)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(PKV_ERR_BAD_BLOCK);
    return;
  }
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < block_chunks;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    k_pool[dst * block_chunks + i] = k_pool[src * block_chunks + i];
    v_pool[dst * block_chunks + i] = v_pool[src * block_chunks + i];
  }
}

// ---------------------------------------------------------------------------
// KV append into e4m3 pools: each thread quantises 8 elements of one (token,
// head) row, x * (1 / scale) in fp32, rounded to nearest e4m3 (ties to even,
// saturating to +-448), and stores 8 bytes.
// ---------------------------------------------------------------------------
template <typename Src>
__device__ __forceinline__ void load8_f32(const Src* p, float (&x)[8]);

template <>
__device__ __forceinline__ void load8_f32<float>(const float* p, float (&x)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

template <>
__device__ __forceinline__ void load8_f32<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 r = *reinterpret_cast<const uint4*>(p);
  float2 f[4];
  Elem<__nv_bfloat16>::widen(r, f);
#pragma unroll
  for (int i = 0; i < 4; ++i) { x[2 * i] = f[i].x; x[2 * i + 1] = f[i].y; }
}

template <>
__device__ __forceinline__ void load8_f32<__half>(const __half* p, float (&x)[8]) {
  const uint4 r = *reinterpret_cast<const uint4*>(p);
  float2 f[4];
  Elem<__half>::widen(r, f);
#pragma unroll
  for (int i = 0; i < 4; ++i) { x[2 * i] = f[i].x; x[2 * i + 1] = f[i].y; }
}

template <typename Src>
__device__ __forceinline__ void append_fp8_group(const AppendArgs& a, int64_t i) {
  const Src* __restrict__ k_new = static_cast<const Src*>(a.k_new);
  const Src* __restrict__ v_new = static_cast<const Src*>(a.v_new);
  const int32_t per_row = a.row_units, num_kv_heads = a.num_kv_heads;
  const int32_t head_dim = per_row * 8;
  const int32_t grp = static_cast<int32_t>(i % per_row);
  const int64_t row = i / per_row;  // token * num_kv_heads + head
  const int32_t h = static_cast<int32_t>(row % num_kv_heads);
  const int64_t tok = row / num_kv_heads;
  const int32_t slot = a.slots[tok];
  if (slot < 0) return;
  const AppendDst t = append_dst(a, tok);
  uint8_t* __restrict__ k_pool = t.k_pool;
  uint8_t* __restrict__ v_pool = t.v_pool;
  const int32_t block_size = t.block_size;
  const int32_t blk = slot / block_size, off = slot - blk * block_size;
  if (blk >= t.num_blocks) {
    if (grp == 0 && h == 0) record_error(PKV_ERR_BAD_BLOCK);
    return;
  }
  const int64_t dst = ((static_cast<int64_t>(blk) * num_kv_heads + h) * block_size + off) * head_dim + grp * 8;
  const int64_t src = row * head_dim + grp * 8;
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    float x[8];
    load8_f32<Src>((kv ? v_new : k_new) + src, x);
    const float inv = kv ? a.v_inv : a.k_inv;
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_fp8x2_storage_t q2 =
          __nv_cvt_float2_to_fp8x2(make_float2(x[2 * j] * inv, x[2 * j + 1] * inv), __NV_SATFINITE, __NV_E4M3);
      packed[j >> 1] |= static_cast<uint32_t>(q2) << (16 * (j & 1));
    }
    *reinterpret_cast<uint2*>((kv ? v_pool : k_pool) + dst) = make_uint2(packed[0], packed[1]);
  }
}

template <typename Src>
__global__ void __launch_bounds__(256) kv_append_fp8_kernel(const AppendArgs a) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < a.n_units) append_fp8_group<Src>(a, i);
}

// ---------------------------------------------------------------------------
// Append and plan in one launch, ahead of the decode kernel of the same step:
// CTA 0 builds the decode work list (plan_body), CTAs 1 .. write the new K/V
// rows into their slots.  The decode kernel waits for the whole grid
// (griddepcontrol.wait) before its first read, so it sees every new row.
// Src = void: 16-byte row copies; otherwise the source type quantised to e4m3.
// ---------------------------------------------------------------------------
template <typename Src>
__global__ void __launch_bounds__(256) append_plan_kernel(const AppendArgs a, const PlanArgs pa,
                                                          int4* __restrict__ items, int32_t* __restrict__ n_items) {
  // launched programmatically serialised: the previous kernel of the stream
  // (which may have produced the new rows, slots or lengths) is complete
  // before anything is read or written
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (blockIdx.x == 0) {
    extern __shared__ int32_t hist[];
    plan_body(pa, items, n_items, hist);
    return;
  }
  const int64_t i = static_cast<int64_t>(blockIdx.x - 1) * blockDim.x + threadIdx.x;
  if (i >= a.n_units) return;
  if constexpr (std::is_void_v<Src>) {
    append_chunk(a, i);
  } else {
    append_fp8_group<Src>(a, i);
  }
}

}  // namespace pkv
