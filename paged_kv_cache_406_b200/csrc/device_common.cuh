// Device-side building blocks for sm_100a: the device status word, bounded
// mbarrier waits, 1-D bulk (TMA) copies into shared memory, and widening of
// 16-byte vectors of f32 / bf16 / f16 elements to fp32 pairs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "paged_kv.h"

namespace pkv {

// First error a kernel recorded since the host last cleared it (PKV_OK if
// none).  One word per device, in this library's own device memory.  All
// kernels live in one translation unit (pkv_device.cu), which owns it.
__device__ int g_status = PKV_OK;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_status, PKV_OK, code); }

// A wait on an mbarrier gives up after this long and reports
// PKV_ERR_DEVICE_TIMEOUT; a healthy copy completes in microseconds.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `bar` with the given parity to complete.  Gives up
// (returns false) once *abort becomes non-zero or after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
  }
}

// 1-D bulk copy global -> this CTA's shared memory, completing `bytes`
// transaction bytes on `bar`.  Both addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// L2 policy for data read exactly once (K/V tiles): evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- element traits: a 16-byte chunk widened to fp32 pairs ----------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kVec = 4;  // elements per 16-byte chunk
  __device__ __forceinline__ static void widen(const uint4& c, float2* f) {
    f[0] = make_float2(__uint_as_float(c.x), __uint_as_float(c.y));
    f[1] = make_float2(__uint_as_float(c.z), __uint_as_float(c.w));
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kVec = 8;
  // bf16 is the high half of an fp32: shifting it into place is exact.
  __device__ __forceinline__ static float2 pair(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
  __device__ __forceinline__ static void widen(const uint4& c, float2* f) {
    f[0] = pair(c.x);
    f[1] = pair(c.y);
    f[2] = pair(c.z);
    f[3] = pair(c.w);
  }
};

template <>
struct Elem<__half> {
  static constexpr int kVec = 8;
  __device__ __forceinline__ static float2 pair(uint32_t w) {
    __half2 h = *reinterpret_cast<const __half2*>(&w);
    return __half22float2(h);
  }
  __device__ __forceinline__ static void widen(const uint4& c, float2* f) {
    f[0] = pair(c.x);
    f[1] = pair(c.y);
    f[2] = pair(c.z);
    f[3] = pair(c.w);
  }
};

}  // namespace pkv
