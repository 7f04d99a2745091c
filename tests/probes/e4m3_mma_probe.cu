// Checks two properties of the fifth-generation tensor cores that the e4m3
// decode kernel (decode_tc8.cuh) relies on, with one CTA and two sequences
// of four tcgen05.mma kind::f8f6f4 instructions (M 128, N 16, K 128 in all):
//   * the operand layouts it uses give the right products: A and B K-major
//     with the 128-byte swizzle (the K tile and the q terms); A MN-major with
//     the 128-byte swizzle and B MN-major without swizzle (V as stored, and
//     the P terms as 16-byte token rows);
//   * e4m3 x e4m3 products are accumulated to fp32 precision.
// For three input sets (full-range random codes; codes in [0.5, 4); one 448 x
// 448 product per output next to small ones) it prints one JSON line per set
// with the largest error against the exact sum, in fp32 ulps of sum |a b|.
// Every wait is bounded (1 s); the program exits non-zero on any CUDA error.
#include <cstdio>
#include <cstdint>
#include <cstdlib>
#include <cmath>
#include <vector>
#include <random>
#include <cuda_runtime.h>

__device__ int g_err = 0;

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}

__host__ __device__ constexpr uint32_t idesc_f8(bool a_mn, bool b_mn, int m, int n) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_f8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}"
               :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

// inputs (host logical layouts): A1[128][128] (m, k), B1[16][128] (n, k), A2[128][128] (k, m), B2[128][16] (k, n)
__global__ void __launch_bounds__(128) probe(const uint8_t* A1, const uint8_t* B1, const uint8_t* A2,
                                             const uint8_t* B2, float* D1, float* D2) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA1 = base;            // 16384
  uint8_t* sB1 = base + 16384;    // 2048
  uint8_t* sA2 = base + 18432;    // 16384
  uint8_t* sB2 = base + 34816;    // 2048
  uint64_t* bar = (uint64_t*)(base + 36864);
  uint32_t* tslot = (uint32_t*)(base + 36872);
  const int t = threadIdx.x;
  // swizzled 128-byte rows: chunk c of row r at c ^ (r % 8)
  for (int i = t; i < 128 * 128; i += 128) {
    const int r = i / 128, c = i % 128;
    sA1[r * 128 + (((c >> 4) ^ (r & 7)) << 4) + (c & 15)] = A1[i];
    sA2[r * 128 + (((c >> 4) ^ (r & 7)) << 4) + (c & 15)] = A2[i];
  }
  for (int i = t; i < 16 * 128; i += 128) {
    const int r = i / 128, c = i % 128;
    sB1[r * 128 + (((c >> 4) ^ (r & 7)) << 4) + (c & 15)] = B1[i];
  }
  for (int i = t; i < 128 * 16; i += 128) sB2[i] = B2[i];  // token k at 16 k
  if (t == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(smem_u32(bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (t < 32) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 32;" :: "r"(smem_u32(tslot)) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;
  if (t == 0) {
    const uint32_t i1 = idesc_f8(false, false, 128, 16), i2 = idesc_f8(true, true, 128, 16);
    for (int ks = 0; ks < 4; ++ks) {
      mma_f8(tmem, desc(smem_u32(sA1) + 32 * ks, 16, 1024, 2), desc(smem_u32(sB1) + 32 * ks, 16, 1024, 2), i1, ks);
    }
    for (int ks = 0; ks < 4; ++ks) {
      mma_f8(tmem + 16, desc(smem_u32(sA2) + 4096 * ks, 16, 1024, 2), desc(smem_u32(sB2) + 512 * ks, 128, 2048, 0), i2, ks);
    }
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
  }
  // bounded wait for the MMAs
  uint32_t ok = 0;
  unsigned long long t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n selp.u32 %0, 1, 0, p;\n}"
                 : "=r"(ok) : "r"(smem_u32(bar)) : "memory");
    if (ok) break;
    unsigned long long t1;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
    if (t1 - t0 > 1000000000ull) break;
  }
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (!ok) {
    if (t == 0) atomicExch(&g_err, 1);
  } else {
    const int w = t / 32;
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(tmem + ((uint32_t)(w * 32) << 16))
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    for (int j = 0; j < 16; ++j) {
      D1[t * 16 + j] = __uint_as_float(r[j]);
      D2[t * 16 + j] = __uint_as_float(r[16 + j]);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (t < 32) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 32;" :: "r"(tmem) : "memory");
}

static double e4m3(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  const double v = e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

int main() {
  std::mt19937 rng(12345);
  auto code = [&](int mode) -> uint8_t {
    uint8_t c = (uint8_t)(rng() & 0xFF);
    if (mode == 1) c = (uint8_t)((rng() & 0x80) | (0x30 + rng() % 0x18));  // about [0.5, 4)
    if ((c & 0x7F) == 0x7F) c ^= 1;
    return c;
  };
  for (int mode = 0; mode < 3; ++mode) {
    std::vector<uint8_t> A1(128 * 128), B1(16 * 128), A2(128 * 128), B2(128 * 16);
    for (auto& c : A1) c = code(mode == 2 ? 1 : mode);
    for (auto& c : B1) c = code(mode == 2 ? 1 : mode);
    for (auto& c : A2) c = code(mode == 2 ? 1 : mode);
    for (auto& c : B2) c = code(mode == 2 ? 1 : mode);
    if (mode == 2) {  // one huge product per output plus small ones: are the small ones kept?
      for (int m = 0; m < 128; ++m) A1[m * 128] = 0x7E;         // 448
      for (int n = 0; n < 16; ++n) B1[n * 128] = 0x7E;
      for (int m = 0; m < 128; ++m) A2[0 * 128 + m] = 0x7E;     // k = 0 row of A2
      for (int n = 0; n < 16; ++n) B2[0 * 16 + n] = 0x7E;
    }
    uint8_t *dA1, *dB1, *dA2, *dB2;
    float *dD1, *dD2;
    cudaMalloc(&dA1, A1.size()); cudaMalloc(&dB1, B1.size()); cudaMalloc(&dA2, A2.size()); cudaMalloc(&dB2, B2.size());
    cudaMalloc(&dD1, 128 * 16 * 4); cudaMalloc(&dD2, 128 * 16 * 4);
    cudaMemcpy(dA1, A1.data(), A1.size(), cudaMemcpyHostToDevice);
    cudaMemcpy(dB1, B1.data(), B1.size(), cudaMemcpyHostToDevice);
    cudaMemcpy(dA2, A2.data(), A2.size(), cudaMemcpyHostToDevice);
    cudaMemcpy(dB2, B2.data(), B2.size(), cudaMemcpyHostToDevice);
    cudaMemset(dD1, 0, 128 * 16 * 4); cudaMemset(dD2, 0, 128 * 16 * 4);
    const int smem = 36864 + 64 + 1024;
    cudaFuncSetAttribute(probe, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    probe<<<1, 128, smem>>>(dA1, dB1, dA2, dB2, dD1, dD2);
    cudaError_t e = cudaDeviceSynchronize();
    int err = 0;
    cudaMemcpyFromSymbol(&err, g_err, sizeof(int));
    if (e != cudaSuccess || err) {
      printf("set %d: %s, timeout flag %d\n", mode, cudaGetErrorString(e), err);
      return 1;
    }
    std::vector<float> D1(128 * 16), D2(128 * 16);
    cudaMemcpy(D1.data(), dD1, D1.size() * 4, cudaMemcpyDeviceToHost);
    cudaMemcpy(D2.data(), dD2, D2.size() * 4, cudaMemcpyDeviceToHost);
    double w1 = 0, w2 = 0, r1 = 0, r2 = 0;
    int exact1 = 0, exact2 = 0;
    for (int m = 0; m < 128; ++m)
      for (int n = 0; n < 16; ++n) {
        double s1 = 0, a1 = 0, s2 = 0, a2 = 0;
        for (int k = 0; k < 128; ++k) {
          const double p1 = e4m3(A1[m * 128 + k]) * e4m3(B1[n * 128 + k]);
          const double p2 = e4m3(A2[k * 128 + m]) * e4m3(B2[k * 16 + n]);
          s1 += p1; a1 += std::fabs(p1); s2 += p2; a2 += std::fabs(p2);
        }
        const double e1 = std::fabs(D1[m * 16 + n] - s1), e2 = std::fabs(D2[m * 16 + n] - s2);
        exact1 += (float)s1 == D1[m * 16 + n];
        exact2 += (float)s2 == D2[m * 16 + n];
        w1 = std::max(w1, e1 / (a1 * std::ldexp(1.0, -23)));
        w2 = std::max(w2, e2 / (a2 * std::ldexp(1.0, -23)));
        r1 = std::max(r1, e1 / a1);
        r2 = std::max(r2, e2 / a2);
      }
    printf("{\"set\": %d, \"kmajor_ulps\": %.4f, \"mnmajor_ulps\": %.4f, \"kmajor_exact\": %d, \"mnmajor_exact\": %d}\n",
           mode, w1, w2, exact1, exact2);
    cudaFree(dA1); cudaFree(dB1); cudaFree(dA2); cudaFree(dB2); cudaFree(dD1); cudaFree(dD2);
  }
  return 0;
}
