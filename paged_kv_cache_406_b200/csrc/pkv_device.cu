// Device entry points of libpagedkv (sm_100a): KV append, block copy,
// PagedAttention decode (plan, decode and partition-merge kernels), append and
// decode in one call, paged prefill, the one-call step from host buffers and
// the device status word.  The kernels live in the .cuh files.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cuda_fp8.h>
#include <nvtx3/nvToolsExt.h>

#include "append.cuh"
#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_tc8.cuh"
#include "device_common.cuh"
#include "prefill.cuh"
#include "pkv_internal.h"

// ===========================================================================
// host side
// ===========================================================================
namespace {

using pkv::fail;

// An NVTX range around one library call, so that a profiler's timeline shows
// each step and each entry point by name (a no-op without a tool attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kMaxDevices = 64;
constexpr int kAutoPartitionTokens = 512;
constexpr int kMaxPartitionTokens = 8192;

size_t elem_size(int dtype) { return dtype == PKV_F32 ? 4 : (dtype == PKV_FP8_E4M3 ? 1 : 2); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_fail(cudaError_t e, const char* what) {
  return fail(PKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int check_common(int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t dtype, const char* fn) {
  if (dtype != PKV_F32 && dtype != PKV_BF16 && dtype != PKV_F16)
    return fail(PKV_ERR_UNSUPPORTED, "%s: dtype %d not supported", fn, dtype);
  if (head_dim != 64 && head_dim != 128)
    return fail(PKV_ERR_UNSUPPORTED, "%s: head_dim %d not supported (64 or 128)", fn, head_dim);
  if (block_size != 8 && block_size != 16 && block_size != 32)
    return fail(PKV_ERR_UNSUPPORTED, "%s: block_size %d not supported (8, 16 or 32)", fn, block_size);
  if (num_kv_heads <= 0) return fail(PKV_ERR_INVALID_ARG, "%s: num_kv_heads %d <= 0", fn, num_kv_heads);
  return PKV_OK;
}

int sm_count(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < kMaxDevices) {
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

int resolve_partition(int32_t partition_tokens, int32_t block_size, int32_t* out) {
  int32_t pt = partition_tokens == 0 ? kAutoPartitionTokens : partition_tokens;
  if (pt < block_size || pt % block_size != 0 || pt > kMaxPartitionTokens)
    return fail(PKV_ERR_INVALID_ARG,
                "partition_tokens %d must be a positive multiple of block_size %d and at most %d",
                partition_tokens, block_size, kMaxPartitionTokens);
  *out = pt;
  return PKV_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  int32_t max_parts;
  size_t items, m, l, o, total;  // byte offsets; n_items lives at offset 0
};

WsLayout ws_layout(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim, int64_t max_tokens,
                   int32_t pt) {
  WsLayout w;
  w.max_parts = static_cast<int32_t>(std::max<int64_t>(1, (max_tokens + pt - 1) / pt));
  const int64_t rows = num_seqs * num_q_heads * w.max_parts;
  w.items = 256;
  (void)num_kv_heads;
  w.m = w.items + round256(num_seqs * w.max_parts * sizeof(int4));
  w.l = w.m + round256(rows * sizeof(float));
  w.o = w.l + round256(rows * sizeof(float));
  w.total = w.o + round256(rows * head_dim * sizeof(float));
  return w;
}

int ring_stages(size_t stage_bytes) {
  // about 64 KB of K/V in flight per CTA; a multiple of the consumer warps
  int ns = static_cast<int>((64 * 1024) / stage_bytes);
  ns = std::max(pkv::kConsumerWarps, std::min(16, ns));
  return ns - ns % pkv::kConsumerWarps;
}

// Launches `kern` with programmatic stream serialisation: the grid may be
// scheduled while the previous kernel in the stream runs; it waits for that
// kernel's results with griddepcontrol.wait before reading them.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// New K/V rows to write in the same launch as the plan kernel (the append of
// a decode step), already checked by the caller.  src_dtype < 0: 16-byte row
// copies into a 16-bit or fp32 pool; otherwise the source dtype of rows
// quantised into an e4m3 pool.
struct PendingAppend {
  pkv::AppendArgs args;
  int src_dtype;
};

// Test support for the decode kernels' bounded waits (pkv_debug_stall_decode):
// a CTA whose first work unit gets no copies.
std::atomic<int> g_stall_cta{-1};
// the same for the prefill kernel (pkv_debug_stall_prefill)
std::atomic<int> g_stall_prefill_cta{-1};

void apply_debug(pkv::DecodeParams& p) { p.stall_cta = g_stall_cta.load(std::memory_order_relaxed); }

// The one pool of a single-pool batch.
void set_single_pool(pkv::DecodeParams& p, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                     int32_t num_blocks, int32_t max_blocks, int32_t block_size) {
  p.pool[0] = pkv::PoolView{k_pool, v_pool, block_tables, num_blocks, max_blocks, block_size, 0};
  p.n_pools = 1;
}

// Append arguments for rows that all go into one pool.
pkv::AppendArgs single_append(const void* k_new, const void* v_new, const int32_t* slots, int64_t n_units,
                              void* k_pool, void* v_pool, int32_t num_blocks, int32_t num_kv_heads,
                              int32_t row_units, int32_t block_size, float k_inv, float v_inv) {
  pkv::AppendArgs a{};
  a.k_new = k_new;
  a.v_new = v_new;
  a.slots = slots;
  a.n_units = n_units;
  a.k_pool[0] = k_pool;
  a.v_pool[0] = v_pool;
  a.num_blocks[0] = num_blocks;
  a.block_size[0] = block_size;
  a.n_pools = 1;
  a.num_kv_heads = num_kv_heads;
  a.row_units = row_units;
  a.k_inv = k_inv;
  a.v_inv = v_inv;
  return a;
}

// Plan arguments of a batch: the sort bins are blocks of a single pool, or
// 16-token chunks when the pools' block sizes differ.
pkv::PlanArgs plan_args(const pkv::DecodeParams& p, const int32_t* seq_lens, int32_t num_seqs) {
  pkv::PlanArgs a{};
  a.seq_lens = seq_lens;
  a.num_seqs = num_seqs;
  a.part_tokens = p.partition_tokens;
  a.bin_tokens = p.n_pools == 1 ? p.pool[0].block_size : pkv::kChunkTokens;
  a.n_pools = p.n_pools;
  for (int c = 0; c < p.n_pools; ++c) {
    a.seq0[c] = p.pool[c].seq0;
    a.cap[c] = p.pool[c].max_blocks * p.pool[c].block_size;
  }
  return a;
}

// plan kernel (or append + plan) -> decode kernel -> merge kernel (the last
// only when some sequence can span more than one partition)
template <int D, typename Kernel, typename... Args>
int launch_plan_decode_merge(const pkv::DecodeParams& p, const int32_t* seq_lens, int32_t num_seqs,
                             int32_t max_tokens, const PendingAppend* ap, Kernel kern, int grid, int threads,
                             size_t smem, cudaStream_t stream, Args... args) {
  const pkv::PlanArgs pa = plan_args(p, seq_lens, num_seqs);
  const int kmax = pa.part_tokens / pa.bin_tokens;
  const size_t plan_smem = 2 * (kmax + 1) * sizeof(int32_t);
  int4* items = const_cast<int4*>(p.items);
  int32_t* n_items = const_cast<int32_t*>(p.n_items);
  // The plan (or append + plan) launch, too, is programmatically serialised:
  // its CTAs are scheduled while the previous kernel of the stream finishes
  // and wait for it (griddepcontrol.wait) before touching memory; this took
  // 2 µs off a 101.5 µs Llama-3-8B-shaped step and 1.7 µs off a 31.4 µs one.
  cudaError_t e = cudaSuccess;
  if (ap) {
    const dim3 g(static_cast<unsigned>(1 + (ap->args.n_units + 255) / 256));
    switch (ap->src_dtype) {
      case -1: e = launch_pdl(pkv::append_plan_kernel<void>, g, dim3(256), plan_smem, stream, ap->args, pa, items, n_items); break;
      case PKV_F32:
        e = launch_pdl(pkv::append_plan_kernel<float>, g, dim3(256), plan_smem, stream, ap->args, pa, items, n_items);
        break;
      case PKV_BF16:
        e = launch_pdl(pkv::append_plan_kernel<__nv_bfloat16>, g, dim3(256), plan_smem, stream, ap->args, pa, items,
                       n_items);
        break;
      default:
        e = launch_pdl(pkv::append_plan_kernel<__half>, g, dim3(256), plan_smem, stream, ap->args, pa, items, n_items);
    }
  } else {
    e = launch_pdl(pkv::plan_kernel, dim3(1), dim3(1024), plan_smem, stream, pa, items, n_items);
  }
  if (e != cudaSuccess) return cuda_fail(e, "plan launch");
  e = launch_pdl(kern, dim3(grid), dim3(threads), smem, stream, p, args...);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  if (p.max_parts > 1) {
    // a warp per (sequence, query head), or a CTA when a sequence can span
    // more than 32 partitions
    const int rows = num_seqs * p.num_q_heads;
    const bool wide = p.max_parts > 32;
    e = launch_pdl(wide ? pkv::merge_wide_kernel<D> : pkv::merge_kernel<D>, dim3(wide ? rows : (rows + 7) / 8),
                   dim3(256), 0, stream, seq_lens, num_seqs, p.num_q_heads, max_tokens, p.partition_tokens,
                   p.max_parts, static_cast<const float*>(p.part_m), static_cast<const float*>(p.part_l),
                   static_cast<const float*>(p.part_o), p.out);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return pkv::ok();
}

template <typename T, int D, int G>
int launch_decode(const pkv::DecodeParams& base, const int32_t* seq_lens, int32_t num_seqs, int32_t max_tokens,
                  const PendingAppend* ap, cudaStream_t stream) {
  pkv::DecodeParams p = base;
  apply_debug(p);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const int32_t bs = p.pool[0].block_size;
  p.n_stages = ring_stages(size_t(2) * bs * D * sizeof(T));
  const size_t smem = pkv::DecodeSmem<T, D, G>::bytes(bs, p.n_stages);
  auto kern = pkv::decode_kernel<T, D, G>;
  auto kern_stall = pkv::decode_kernel<T, D, G, true>;

  // per device: opt in to the largest dynamic shared memory any block size
  // needs (once), then cache resident CTAs per SM for this block size
  static std::atomic<int> occ_cache[kMaxDevices][3];
  const int bs_idx = bs == 8 ? 0 : (bs == 16 ? 1 : 2);
  int occ = dev < kMaxDevices ? occ_cache[dev][bs_idx].load(std::memory_order_relaxed) : 0;
  if (occ == 0) {
    size_t smem_max = 0;
    for (int bs : {8, 16, 32})
      smem_max = std::max(smem_max, pkv::DecodeSmem<T, D, G>::bytes(bs, ring_stages(size_t(2) * bs * D * sizeof(T))));
    for (auto k : {kern, kern_stall}) {
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_max));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
      e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(carveout)");
    }
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, pkv::kDecodeThreads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (occ <= 0) return fail(PKV_ERR_CUDA, "decode kernel does not fit on an SM (smem %zu)", smem);
    if (dev < kMaxDevices) occ_cache[dev][bs_idx].store(occ, std::memory_order_relaxed);
  }

  const int64_t work_upper = int64_t(num_seqs) * p.max_parts * p.num_kv_heads;
  const int grid = static_cast<int>(std::min<int64_t>(int64_t(sm_count(dev)) * occ, work_upper));
  return launch_plan_decode_merge<D>(p, seq_lens, num_seqs, max_tokens, ap, p.stall_cta >= 0 ? kern_stall : kern,
                                     grid, pkv::kDecodeThreads, smem, stream);
}

// ---- tensor maps over the K/V pools for the tensor-core kernel ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Pool viewed as a 3-D tensor of 16-bit elements: x = 64 elements (one 128-byte
// column half), y = token row (num_blocks * Hkv * block_size rows, head_dim * 2
// bytes apart), z = column half (head_dim / 64 of them, 128 bytes apart).  A
// box of 64 x box_rows x halves lands in shared memory as [half][row][128 B]
// with 128-byte swizzle.
int make_pool_map(CUtensorMap* m, const void* pool, int dtype, int64_t rows, int head_dim, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (dtype == PKV_FP8_E4M3) {
    // e4m3 codes: a row of head_dim bytes is one box column (head_dim = 128: 128 B)
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows), 1};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(head_dim)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(head_dim), static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(pool), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled (e4m3) failed (%d)", static_cast<int>(r));
    return PKV_OK;
  }
  const cuuint32_t halves = static_cast<cuuint32_t>(head_dim / 64);
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), halves};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2, 128};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), halves};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                   const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return PKV_OK;
}

// Small cache of encoded maps: a decode step reuses the same pools every call
// (up to 16 pools' K and V maps: several caches, or several block-size pools).
struct MapCacheEntry {
  const void* pool;
  int64_t rows;
  int dtype, head_dim, box_rows;
  CUtensorMap map;
};

int pool_map(CUtensorMap* out, const void* pool, int dtype, int64_t rows, int head_dim, int box_rows) {
  static std::mutex mu;
  static MapCacheEntry cache[16];
  static int next = 0, used = 0;
  std::lock_guard<std::mutex> g(mu);
  for (int i = 0; i < used; ++i) {
    const MapCacheEntry& e = cache[i];
    if (e.pool == pool && e.rows == rows && e.dtype == dtype && e.head_dim == head_dim && e.box_rows == box_rows) {
      *out = e.map;
      return PKV_OK;
    }
  }
  int rc = make_pool_map(out, pool, dtype, rows, head_dim, box_rows);
  if (rc) return rc;
  cache[next] = MapCacheEntry{pool, rows, dtype, head_dim, box_rows, *out};
  next = (next + 1) % 16;
  used = used < 16 ? used + 1 : 16;
  return PKV_OK;
}

template <typename T, int D, int G, bool kMulti = false>
int launch_decode_mma(const pkv::DecodeParams& base, const int32_t* seq_lens, int32_t num_seqs, int32_t max_tokens,
                      int dtype, const PendingAppend* ap, cudaStream_t stream) {
  pkv::DecodeParams p = base;
  apply_debug(p);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  using Smem = pkv::MmaSmem<T, D, G>;
  p.n_stages = 8;
  const size_t smem = Smem::bytes(p.n_stages);
  auto kern = pkv::decode_mma_kernel<T, D, G, kMulti>;
  // the bounded-wait test instance exists for single-pool batches only
  auto kern_stall = pkv::decode_mma_kernel<T, D, G, kMulti, !kMulti>;
  static std::atomic<int> occ_cache[kMaxDevices];
  int occ = dev < kMaxDevices ? occ_cache[dev].load(std::memory_order_relaxed) : 0;
  if (occ == 0) {
    for (auto k : {kern, kern_stall}) {
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_mma)");
      e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(carveout)");
    }
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, Smem::kThreads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (occ <= 0) return fail(PKV_ERR_CUDA, "decode_mma kernel does not fit on an SM (smem %zu)", smem);
    if (dev < kMaxDevices) occ_cache[dev].store(occ, std::memory_order_relaxed);
  }
  pkv::PoolMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  for (int c = 0; c < p.n_pools; ++c) {
    const pkv::PoolView& pv = p.pool[c];
    const int64_t rows = int64_t(pv.num_blocks) * p.num_kv_heads * pv.block_size;
    const int box_rows = pv.block_size < pkv::kChunkTokens ? pv.block_size : pkv::kChunkTokens;
    int rc = pool_map(&maps.k[c], pv.k, dtype, rows, D, box_rows);
    if (rc) return rc;
    rc = pool_map(&maps.v[c], pv.v, dtype, rows, D, box_rows);
    if (rc) return rc;
  }

  const int64_t work_upper = int64_t(num_seqs) * p.max_parts * p.num_kv_heads;
  const int grid = static_cast<int>(std::min<int64_t>(int64_t(sm_count(dev)) * occ, work_upper));
  return launch_plan_decode_merge<D>(p, seq_lens, num_seqs, max_tokens, ap, p.stall_cta >= 0 ? kern_stall : kern,
                                     grid, Smem::kThreads, smem, stream, maps);
}

template <typename T>
int dispatch_decode_mma(int32_t head_dim, int32_t group, const pkv::DecodeParams& p, const int32_t* seq_lens,
                        int32_t num_seqs, int32_t max_tokens, int dtype, const PendingAppend* ap, cudaStream_t s) {
  if (head_dim == 128) {
    if (group == 2) return launch_decode_mma<T, 128, 2>(p, seq_lens, num_seqs, max_tokens, dtype, ap, s);
    if (group == 4) return launch_decode_mma<T, 128, 4>(p, seq_lens, num_seqs, max_tokens, dtype, ap, s);
    return launch_decode_mma<T, 128, 8>(p, seq_lens, num_seqs, max_tokens, dtype, ap, s);
  }
  if (group == 2) return launch_decode_mma<T, 64, 2>(p, seq_lens, num_seqs, max_tokens, dtype, ap, s);
  if (group == 4) return launch_decode_mma<T, 64, 4>(p, seq_lens, num_seqs, max_tokens, dtype, ap, s);
  return launch_decode_mma<T, 64, 8>(p, seq_lens, num_seqs, max_tokens, dtype, ap, s);
}

template <typename T>
int dispatch_decode(int32_t head_dim, int32_t group, const pkv::DecodeParams& p, const int32_t* seq_lens,
                    int32_t num_seqs, int32_t max_tokens, const PendingAppend* ap, cudaStream_t s) {
  if (head_dim == 128) {
    if (group == 1) return launch_decode<T, 128, 1>(p, seq_lens, num_seqs, max_tokens, ap, s);
    if (group == 2) return launch_decode<T, 128, 2>(p, seq_lens, num_seqs, max_tokens, ap, s);
    return launch_decode<T, 128, 4>(p, seq_lens, num_seqs, max_tokens, ap, s);
  }
  if (group == 1) return launch_decode<T, 64, 1>(p, seq_lens, num_seqs, max_tokens, ap, s);
  if (group == 2) return launch_decode<T, 64, 2>(p, seq_lens, num_seqs, max_tokens, ap, s);
  return launch_decode<T, 64, 4>(p, seq_lens, num_seqs, max_tokens, ap, s);
}

}  // namespace

extern "C" int pkv_kv_append(const void* k_new, const void* v_new, const int32_t* slot_mapping, int32_t n_tokens,
                             void* k_pool, void* v_pool, int32_t num_blocks, int32_t num_kv_heads,
                             int32_t head_dim, int32_t block_size, int32_t dtype, void* stream) {
  NvtxRange nvtx_range("pkv_kv_append");
  int rc = check_common(num_kv_heads, head_dim, block_size, dtype, "pkv_kv_append");
  if (rc) return rc;
  if (n_tokens < 0 || num_blocks <= 0) return fail(PKV_ERR_INVALID_ARG, "pkv_kv_append: n_tokens/num_blocks");
  if (n_tokens == 0) return pkv::ok();
  if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool)
    return fail(PKV_ERR_INVALID_ARG, "pkv_kv_append: NULL pointer");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
    return fail(PKV_ERR_INVALID_ARG, "pkv_kv_append: K/V buffers must be 16-byte aligned");
  const int32_t row_chunks = static_cast<int32_t>(head_dim * elem_size(dtype) / 16);
  const int64_t n_chunks = int64_t(n_tokens) * num_kv_heads * row_chunks;
  const int64_t blocks = (n_chunks + 255) / 256;
  const pkv::AppendArgs a = single_append(k_new, v_new, slot_mapping, n_chunks, k_pool, v_pool, num_blocks,
                                          num_kv_heads, row_chunks, block_size, 1.0f, 1.0f);
  pkv::kv_append_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pkv_kv_append launch");
  return pkv::ok();
}

extern "C" int pkv_copy_blocks(void* k_pool, void* v_pool, const int32_t* block_pairs, int32_t n_pairs,
                               int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int32_t dtype, void* stream) {
  NvtxRange nvtx_range("pkv_copy_blocks");
  // a byte copy: e4m3 pools are copied like 16-bit ones, at one byte per element
  int rc = check_common(num_kv_heads, head_dim, block_size, dtype == PKV_FP8_E4M3 ? PKV_F16 : dtype, "pkv_copy_blocks");
  if (rc) return rc;
  if (n_pairs < 0 || num_blocks <= 0) return fail(PKV_ERR_INVALID_ARG, "pkv_copy_blocks: n_pairs/num_blocks");
  if (n_pairs == 0) return pkv::ok();
  if (n_pairs > 65535) return fail(PKV_ERR_INVALID_ARG, "pkv_copy_blocks: at most 65535 pairs per call");
  if (!k_pool || !v_pool || !block_pairs) return fail(PKV_ERR_INVALID_ARG, "pkv_copy_blocks: NULL pointer");
  if (!aligned16(k_pool) || !aligned16(v_pool))
    return fail(PKV_ERR_INVALID_ARG, "pkv_copy_blocks: pools must be 16-byte aligned");
  const int64_t block_chunks = int64_t(num_kv_heads) * block_size * head_dim * elem_size(dtype) / 16;
  const int64_t xb = std::min<int64_t>((block_chunks + 255) / 256, 64);
  dim3 grid(static_cast<unsigned>(xb), static_cast<unsigned>(n_pairs));
  pkv::copy_blocks_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), block_pairs, num_blocks, block_chunks);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pkv_copy_blocks launch");
  return pkv::ok();
}

extern "C" int pkv_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                         int32_t head_dim, int32_t max_blocks_per_seq, int32_t block_size,
                                         int32_t partition_tokens, size_t* bytes) {
  if (!bytes) return fail(PKV_ERR_INVALID_ARG, "pkv_decode_workspace_size: bytes is NULL");
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_blocks_per_seq < 0 ||
      block_size <= 0)
    return fail(PKV_ERR_INVALID_ARG, "pkv_decode_workspace_size: bad sizes");
  int32_t pt = 0;
  int rc = resolve_partition(partition_tokens, block_size, &pt);
  if (rc) return rc;
  *bytes = ws_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, int64_t(max_blocks_per_seq) * block_size, pt).total;
  return pkv::ok();
}

namespace {

// The new rows alone (a step whose batch is empty).
int launch_append_only(const PendingAppend& ap, cudaStream_t s) {
  const unsigned blocks = static_cast<unsigned>((ap.args.n_units + 255) / 256);
  switch (ap.src_dtype) {
    case -1: pkv::kv_append_kernel<<<blocks, 256, 0, s>>>(ap.args); break;
    case PKV_F32: pkv::kv_append_fp8_kernel<float><<<blocks, 256, 0, s>>>(ap.args); break;
    case PKV_BF16: pkv::kv_append_fp8_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(ap.args); break;
    default: pkv::kv_append_fp8_kernel<__half><<<blocks, 256, 0, s>>>(ap.args);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return pkv::ok();
}

// Decode over 16-bit or fp32 pools; with `ap`, the step's new rows are
// written by the plan launch first.
int decode_16(const char* fn, const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
              const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
              int32_t num_blocks, int32_t max_blocks_per_seq, int32_t block_size, float scale, int32_t dtype,
              int32_t partition_tokens, void* workspace, size_t workspace_bytes, float* out,
              const PendingAppend* ap, void* stream) {
  int rc = check_common(num_kv_heads, head_dim, block_size, dtype, fn);
  if (rc) return rc;
  if (num_seqs < 0 || num_q_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq < 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad sizes", fn);
  if (num_q_heads % num_kv_heads != 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: num_q_heads %d not a multiple of num_kv_heads %d", fn, num_q_heads,
                num_kv_heads);
  const int32_t group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PKV_ERR_UNSUPPORTED, "%s: group size %d not supported (1, 2, 4 or 8)", fn, group);
  if (group == 8 && dtype == PKV_F32)
    return fail(PKV_ERR_UNSUPPORTED, "%s: group size 8 needs 16-bit K/V", fn);
  if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID_ARG, "%s: scale is not finite", fn);
  int32_t pt = 0;
  rc = resolve_partition(partition_tokens, block_size, &pt);
  if (rc) return rc;
  if (num_seqs == 0) return ap ? launch_append_only(*ap, static_cast<cudaStream_t>(stream)) : pkv::ok();
  if (!q || !k_pool || !v_pool || !block_tables || !seq_lens || !workspace || !out)
    return fail(PKV_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return fail(PKV_ERR_INVALID_ARG, "%s: q, pools and out must be 16-byte aligned", fn);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  const int64_t max_tokens = int64_t(max_blocks_per_seq) * block_size;
  if (max_tokens > (int64_t(1) << 30)) return fail(PKV_ERR_INVALID_ARG, "%s: max_blocks_per_seq too large", fn);
  const WsLayout w = ws_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_tokens, pt);
  if (workspace_bytes < w.total)
    return fail(PKV_ERR_INVALID_ARG, "%s: workspace %zu bytes < %zu needed", fn, workspace_bytes, w.total);

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  pkv::DecodeParams p{};
  p.q = q;
  set_single_pool(p, k_pool, v_pool, block_tables, num_blocks, max_blocks_per_seq, block_size);
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.partition_tokens = pt;
  p.max_parts = w.max_parts;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.v_scale = 1.0f;
  p.items = reinterpret_cast<const int4*>(ws + w.items);
  p.n_items = reinterpret_cast<const int32_t*>(ws);
  p.part_m = reinterpret_cast<float*>(ws + w.m);
  p.part_l = reinterpret_cast<float*>(ws + w.l);
  p.part_o = reinterpret_cast<float*>(ws + w.o);
  p.out = out;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t mt = static_cast<int32_t>(max_tokens);
  // 16-bit K/V with grouped heads: tensor-core kernel (16-token chunks);
  // otherwise the CUDA-core kernel
  if (dtype != PKV_F32 && group >= 2 && pt % pkv::kChunkTokens == 0) {
    if (int64_t(num_blocks) * num_kv_heads * block_size > INT32_MAX)
      return fail(PKV_ERR_INVALID_ARG, "%s: pool has more than 2^31 token rows", fn);
    if (dtype == PKV_BF16)
      return dispatch_decode_mma<__nv_bfloat16>(head_dim, group, p, seq_lens, num_seqs, mt, dtype, ap, s);
    return dispatch_decode_mma<__half>(head_dim, group, p, seq_lens, num_seqs, mt, dtype, ap, s);
  }
  if (group == 8) return fail(PKV_ERR_UNSUPPORTED, "%s: group size 8 needs partition_tokens %% 16 == 0", fn);
  switch (dtype) {
    case PKV_F32: return dispatch_decode<float>(head_dim, group, p, seq_lens, num_seqs, mt, ap, s);
    case PKV_BF16: return dispatch_decode<__nv_bfloat16>(head_dim, group, p, seq_lens, num_seqs, mt, ap, s);
    default: return dispatch_decode<__half>(head_dim, group, p, seq_lens, num_seqs, mt, ap, s);
  }
}

}  // namespace

extern "C" int pkv_paged_attention_decode(const void* q, const void* k_pool, const void* v_pool,
                                          const int32_t* block_tables, const int32_t* seq_lens, int32_t num_seqs,
                                          int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                          int32_t num_blocks, int32_t max_blocks_per_seq, int32_t block_size,
                                          float scale, int32_t dtype, int32_t partition_tokens, void* workspace,
                                          size_t workspace_bytes, float* out, void* stream) {
  NvtxRange nvtx_range("pkv_paged_attention_decode");
  return decode_16("pkv_paged_attention_decode", q, k_pool, v_pool, block_tables, seq_lens, num_seqs, num_q_heads,
                   num_kv_heads, head_dim, num_blocks, max_blocks_per_seq, block_size, scale, dtype, partition_tokens,
                   workspace, workspace_bytes, out, nullptr, stream);
}

extern "C" int pkv_append_and_decode(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                                     int32_t n_tokens, const void* q, void* k_pool, void* v_pool,
                                     const int32_t* block_tables, const int32_t* seq_lens, int32_t num_seqs,
                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                                     int32_t max_blocks_per_seq, int32_t block_size, float scale, int32_t dtype,
                                     int32_t partition_tokens, void* workspace, size_t workspace_bytes, float* out,
                                     void* stream) {
  NvtxRange nvtx_range("pkv_append_and_decode");
  const char* fn = "pkv_append_and_decode";
  int rc = check_common(num_kv_heads, head_dim, block_size, dtype, fn);
  if (rc) return rc;
  if (n_tokens < 0 || num_blocks <= 0) return fail(PKV_ERR_INVALID_ARG, "%s: n_tokens/num_blocks", fn);
  if (n_tokens > 0) {
    if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool) return fail(PKV_ERR_INVALID_ARG, "%s: NULL pointer", fn);
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
      return fail(PKV_ERR_INVALID_ARG, "%s: K/V buffers must be 16-byte aligned", fn);
  }
  const int32_t row_chunks = static_cast<int32_t>(head_dim * elem_size(dtype) / 16);
  PendingAppend ap{single_append(k_new, v_new, slot_mapping, int64_t(n_tokens) * num_kv_heads * row_chunks, k_pool,
                                 v_pool, num_blocks, num_kv_heads, row_chunks, block_size, 1.0f, 1.0f),
                   -1};
  return decode_16(fn, q, k_pool, v_pool, block_tables, seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                   num_blocks, max_blocks_per_seq, block_size, scale, dtype, partition_tokens, workspace,
                   workspace_bytes, out, n_tokens > 0 ? &ap : nullptr, stream);
}

extern "C" int pkv_debug_stall_prefill(int32_t cta) {
  g_stall_prefill_cta.store(cta < 0 ? -1 : cta, std::memory_order_relaxed);
  return pkv::ok();
}

extern "C" int pkv_debug_stall_decode(int32_t cta) {
  g_stall_cta.store(cta < 0 ? -1 : cta, std::memory_order_relaxed);
  return pkv::ok();
}

extern "C" int pkv_device_status(void* stream, int32_t* status, int32_t clear) {
  if (!status) return fail(PKV_ERR_INVALID_ARG, "pkv_device_status: status is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pkv_device_status: cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, pkv::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "pkv_device_status: read");
  if (clear) {
    const int zero = PKV_OK;
    e = cudaMemcpyToSymbol(pkv::g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "pkv_device_status: clear");
  }
  *status = v;
  return pkv::ok();
}

// ===========================================================================
// A decode step over a batch spread across pools of different block sizes
// ===========================================================================
namespace {

constexpr int kMaxPoolsAbi = pkv::kMaxPools;

// Checks the pool list; on success `total` is the batch size, `max_tokens`
// the largest per-sequence capacity and `pt` the partition size.
int check_pools(const char* fn, const pkv_pool_t* pools, int32_t n_pools, int32_t partition_tokens, int64_t* total,
                int64_t* max_tokens, int32_t* pt) {
  if (!pools || n_pools < 1 || n_pools > kMaxPoolsAbi)
    return fail(PKV_ERR_INVALID_ARG, "%s: 1 to %d pools", fn, kMaxPoolsAbi);
  int32_t part = partition_tokens == 0 ? kAutoPartitionTokens : partition_tokens;
  if (part <= 0 || part % pkv::kChunkTokens != 0 || part > kMaxPartitionTokens)
    return fail(PKV_ERR_INVALID_ARG, "%s: partition_tokens %d must be a positive multiple of 16, at most %d", fn,
                partition_tokens, kMaxPartitionTokens);
  *total = 0;
  *max_tokens = 0;
  for (int c = 0; c < n_pools; ++c) {
    const pkv_pool_t& q = pools[c];
    if (q.block_size != 8 && q.block_size != 16 && q.block_size != 32)
      return fail(PKV_ERR_UNSUPPORTED, "%s: pool %d block_size %d not supported (8, 16 or 32)", fn, c, q.block_size);
    if (part % q.block_size != 0)
      return fail(PKV_ERR_INVALID_ARG, "%s: partition_tokens %d is not a multiple of pool %d's block_size %d", fn, part,
                  c, q.block_size);
    if (q.num_seqs < 0 || q.num_blocks <= 0 || q.max_blocks_per_seq < 0)
      return fail(PKV_ERR_INVALID_ARG, "%s: pool %d: bad sizes", fn, c);
    *total += q.num_seqs;
    *max_tokens = std::max<int64_t>(*max_tokens, int64_t(q.max_blocks_per_seq) * q.block_size);
  }
  if (*total > INT32_MAX / 2) return fail(PKV_ERR_INVALID_ARG, "%s: too many sequences", fn);
  if (*max_tokens > (int64_t(1) << 30)) return fail(PKV_ERR_INVALID_ARG, "%s: max_blocks_per_seq too large", fn);
  *pt = part;
  return PKV_OK;
}

}  // namespace

extern "C" int pkv_decode_pools_workspace_size(const pkv_pool_t* pools, int32_t n_pools, int32_t num_q_heads,
                                               int32_t num_kv_heads, int32_t head_dim, int32_t partition_tokens,
                                               size_t* bytes) {
  const char* fn = "pkv_decode_pools_workspace_size";
  if (!bytes) return fail(PKV_ERR_INVALID_ARG, "%s: bytes is NULL", fn);
  if (num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0) return fail(PKV_ERR_INVALID_ARG, "%s: bad sizes", fn);
  int64_t total = 0, max_tokens = 0;
  int32_t pt = 0;
  int rc = check_pools(fn, pools, n_pools, partition_tokens, &total, &max_tokens, &pt);
  if (rc) return rc;
  *bytes = ws_layout(total, num_q_heads, num_kv_heads, head_dim, max_tokens, pt).total;
  return pkv::ok();
}

extern "C" int pkv_append_and_decode_pools(const pkv_pool_t* pools, int32_t n_pools, const void* k_new,
                                           const void* v_new, const int32_t* slot_mapping, const void* q,
                                           const int32_t* seq_lens, int32_t num_q_heads, int32_t num_kv_heads,
                                           int32_t head_dim, float scale, int32_t dtype, int32_t partition_tokens,
                                           void* workspace, size_t workspace_bytes, float* out, void* stream) {
  const char* fn = "pkv_append_and_decode_pools";
  NvtxRange nvtx_range(fn);
  if (dtype != PKV_BF16 && dtype != PKV_F16)
    return fail(PKV_ERR_UNSUPPORTED, "%s: dtype %d not supported (bf16 or f16)", fn, dtype);
  if (head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "%s: head_dim %d not supported (128)", fn, head_dim);
  if (num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: num_q_heads %d must be a positive multiple of num_kv_heads %d", fn,
                num_q_heads, num_kv_heads);
  const int32_t group = num_q_heads / num_kv_heads;
  if (group != 2 && group != 4 && group != 8)
    return fail(PKV_ERR_UNSUPPORTED, "%s: group size %d not supported (2, 4 or 8)", fn, group);
  if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID_ARG, "%s: scale is not finite", fn);
  int64_t total = 0, max_tokens = 0;
  int32_t pt = 0;
  int rc = check_pools(fn, pools, n_pools, partition_tokens, &total, &max_tokens, &pt);
  if (rc) return rc;
  if (total == 0) return pkv::ok();
  if (!k_new || !v_new || !slot_mapping || !q || !seq_lens || !workspace || !out)
    return fail(PKV_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(q) || !aligned16(out))
    return fail(PKV_ERR_INVALID_ARG, "%s: q, new rows and out must be 16-byte aligned", fn);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  const int32_t N = static_cast<int32_t>(total);
  const WsLayout w = ws_layout(N, num_q_heads, num_kv_heads, head_dim, max_tokens, pt);
  if (workspace_bytes < w.total)
    return fail(PKV_ERR_INVALID_ARG, "%s: workspace %zu bytes < %zu needed", fn, workspace_bytes, w.total);

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  pkv::DecodeParams p{};
  p.q = q;
  const int32_t row_chunks = head_dim * 2 / 16;
  pkv::AppendArgs a{};
  a.k_new = k_new;
  a.v_new = v_new;
  a.slots = slot_mapping;
  a.n_units = int64_t(N) * num_kv_heads * row_chunks;
  a.n_pools = n_pools;
  a.num_kv_heads = num_kv_heads;
  a.row_units = row_chunks;
  a.k_inv = a.v_inv = 1.0f;
  int32_t seq0 = 0;
  for (int c = 0; c < n_pools; ++c) {
    const pkv_pool_t& pc = pools[c];
    if (pc.num_seqs > 0) {
      if (!pc.k_pool || !pc.v_pool || !pc.block_tables) return fail(PKV_ERR_INVALID_ARG, "%s: pool %d: NULL pointer", fn, c);
      if (!aligned16(pc.k_pool) || !aligned16(pc.v_pool))
        return fail(PKV_ERR_INVALID_ARG, "%s: pool %d must be 16-byte aligned", fn, c);
    }
    if (int64_t(pc.num_blocks) * num_kv_heads * pc.block_size > INT32_MAX)
      return fail(PKV_ERR_INVALID_ARG, "%s: pool %d has more than 2^31 token rows", fn, c);
    p.pool[c] = pkv::PoolView{pc.k_pool, pc.v_pool, pc.block_tables, pc.num_blocks, pc.max_blocks_per_seq,
                              pc.block_size, seq0};
    a.k_pool[c] = pc.k_pool;
    a.v_pool[c] = pc.v_pool;
    a.num_blocks[c] = pc.num_blocks;
    a.block_size[c] = pc.block_size;
    a.tok0[c] = seq0;
    seq0 += pc.num_seqs;
  }
  // pools without sequences still count in the thresholds (seq0 equal to the
  // next pool's), so no sequence maps to them
  p.n_pools = n_pools;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.partition_tokens = pt;
  p.max_parts = w.max_parts;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.v_scale = 1.0f;
  p.items = reinterpret_cast<const int4*>(ws + w.items);
  p.n_items = reinterpret_cast<const int32_t*>(ws);
  p.part_m = reinterpret_cast<float*>(ws + w.m);
  p.part_l = reinterpret_cast<float*>(ws + w.l);
  p.part_o = reinterpret_cast<float*>(ws + w.o);
  p.out = out;
  const PendingAppend ap{a, -1};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t mt = static_cast<int32_t>(max_tokens);
  if (dtype == PKV_BF16) {
    if (group == 2) return launch_decode_mma<__nv_bfloat16, 128, 2, true>(p, seq_lens, N, mt, dtype, &ap, s);
    if (group == 4) return launch_decode_mma<__nv_bfloat16, 128, 4, true>(p, seq_lens, N, mt, dtype, &ap, s);
    return launch_decode_mma<__nv_bfloat16, 128, 8, true>(p, seq_lens, N, mt, dtype, &ap, s);
  }
  if (group == 2) return launch_decode_mma<__half, 128, 2, true>(p, seq_lens, N, mt, dtype, &ap, s);
  if (group == 4) return launch_decode_mma<__half, 128, 4, true>(p, seq_lens, N, mt, dtype, &ap, s);
  return launch_decode_mma<__half, 128, 8, true>(p, seq_lens, N, mt, dtype, &ap, s);
}

// e4m3 pools: the tcgen05 kernel (decode_tc8.cuh), persistent CTAs with a ring
// of 128-token chunks: three CTAs per SM with two stages each (G <= 4), two
// with three (G = 8, whose registers do not fit three CTAs).  On the
// Llama-3-8B batch 3 x 2 stages ran 4.8 % faster than 2 x 3 and 45 % faster
// than one CTA with 6: the softmax warps' latency, not the bytes in flight,
// bounds the kernel, so more of them per SM is what pays.
__host__ __device__ constexpr int tc8_stages(int g) { return g == 8 ? 3 : 2; }

template <int G>
int launch_decode_tc8(const pkv::DecodeParams& base, const int32_t* seq_lens, int32_t num_seqs, int32_t max_tokens,
                      const PendingAppend* ap, cudaStream_t stream) {
  pkv::DecodeParams p = base;
  apply_debug(p);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  constexpr int NSt = tc8_stages(G);
  const size_t smem = pkv::t8::Layout<NSt, G>::kSmemBytes;
  auto kern = pkv::decode_tc8_kernel<G, NSt>;
  auto kern_stall = pkv::decode_tc8_kernel<G, NSt, true>;  // the bounded-wait test instance
  static std::atomic<int> occ_cache[kMaxDevices];
  int occ = dev < kMaxDevices ? occ_cache[dev].load(std::memory_order_relaxed) : 0;
  if (occ == 0) {
    for (auto k : {kern, kern_stall}) {
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_tc8)");
      e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(carveout)");
    }
    // CTAs per SM from the SM's shared memory (the occupancy query counts
    // one CTA where two fit: measured, two are co-resident and run 1.6x as
    // fast); the launch bounds keep the registers of that many CTAs within
    // the SM's file, and each CTA holds 128 of the 512 tensor-memory columns
    int smem_sm = 0, reserved = 0;
    e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(smem per SM)");
    e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(reserved smem)");
    occ = std::min(NSt == 2 ? 3 : 2, smem_sm / static_cast<int>(smem + static_cast<size_t>(reserved)));
    if (occ <= 0) return fail(PKV_ERR_CUDA, "decode_tc8 kernel does not fit on an SM (smem %zu)", smem);
    if (dev < kMaxDevices) occ_cache[dev].store(occ, std::memory_order_relaxed);
  }
  const pkv::PoolView& pv = p.pool[0];
  const int64_t rows = int64_t(pv.num_blocks) * p.num_kv_heads * pv.block_size;
  const int box_rows = pv.block_size < pkv::kChunkTokens ? pv.block_size : pkv::kChunkTokens;
  CUtensorMap mk, mv;
  int rc = pool_map(&mk, pv.k, PKV_FP8_E4M3, rows, pkv::t8::kD, box_rows);
  if (rc) return rc;
  rc = pool_map(&mv, pv.v, PKV_FP8_E4M3, rows, pkv::t8::kD, box_rows);
  if (rc) return rc;
  const int64_t work_upper = int64_t(num_seqs) * p.max_parts * p.num_kv_heads;
  const int grid = static_cast<int>(std::min<int64_t>(int64_t(sm_count(dev)) * occ, work_upper));
  return launch_plan_decode_merge<128>(p, seq_lens, num_seqs, max_tokens, ap, p.stall_cta >= 0 ? kern_stall : kern,
                                       grid, pkv::t8::kThreads, smem, stream, mk, mv);
}

// ===========================================================================
// FP8 (e4m3) KV cache
// ===========================================================================
extern "C" int pkv_kv_append_fp8(const void* k_new, const void* v_new, int32_t src_dtype,
                                 const int32_t* slot_mapping, int32_t n_tokens, void* k_pool, void* v_pool,
                                 int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 float k_scale, float v_scale, void* stream) {
  NvtxRange nvtx_range("pkv_kv_append_fp8");
  const char* fn = "pkv_kv_append_fp8";
  int rc = check_common(num_kv_heads, head_dim, block_size, src_dtype, fn);
  if (rc) return rc;
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return fail(PKV_ERR_INVALID_ARG, "%s: scales must be positive and finite", fn);
  if (n_tokens < 0 || num_blocks <= 0) return fail(PKV_ERR_INVALID_ARG, "%s: n_tokens/num_blocks", fn);
  if (n_tokens == 0) return pkv::ok();
  if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool) return fail(PKV_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
    return fail(PKV_ERR_INVALID_ARG, "%s: buffers must be 16-byte aligned", fn);
  const float k_inv = static_cast<float>(1.0 / static_cast<double>(k_scale));
  const float v_inv = static_cast<float>(1.0 / static_cast<double>(v_scale));
  const int64_t n_groups = int64_t(n_tokens) * num_kv_heads * (head_dim / 8);
  const unsigned blocks = static_cast<unsigned>((n_groups + 255) / 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const pkv::AppendArgs a = single_append(k_new, v_new, slot_mapping, n_groups, k_pool, v_pool, num_blocks,
                                          num_kv_heads, head_dim / 8, block_size, k_inv, v_inv);
  switch (src_dtype) {
    case PKV_F32: pkv::kv_append_fp8_kernel<float><<<blocks, 256, 0, s>>>(a); break;
    case PKV_BF16: pkv::kv_append_fp8_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(a); break;
    default: pkv::kv_append_fp8_kernel<__half><<<blocks, 256, 0, s>>>(a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pkv_kv_append_fp8 launch");
  return pkv::ok();
}

namespace {

int decode_fp8(const char* fn, const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
               const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
               int32_t head_dim, int32_t num_blocks, int32_t max_blocks_per_seq, int32_t block_size, float scale,
               float k_scale, float v_scale, int32_t partition_tokens, void* workspace, size_t workspace_bytes,
               float* out, const PendingAppend* ap, void* stream) {
  int rc = check_common(num_kv_heads, head_dim, block_size, PKV_F16, fn);
  if (rc) return rc;
  if (head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "%s: e4m3 pools need head_dim 128", fn);
  if (num_seqs < 0 || num_q_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq < 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad sizes", fn);
  if (num_q_heads % num_kv_heads != 0) return fail(PKV_ERR_INVALID_ARG, "%s: num_q_heads % num_kv_heads != 0", fn);
  const int32_t group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PKV_ERR_UNSUPPORTED, "%s: group size %d not supported (1, 2, 4 or 8)", fn, group);
  if (!std::isfinite(scale) || !(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
      !std::isfinite(v_scale))
    return fail(PKV_ERR_INVALID_ARG, "%s: scale must be finite and k_scale, v_scale positive", fn);
  int32_t pt = 0;
  rc = resolve_partition(partition_tokens, block_size, &pt);
  if (rc) return rc;
  if (pt % pkv::kChunkTokens != 0) return fail(PKV_ERR_INVALID_ARG, "%s: partition_tokens must be a multiple of 16", fn);
  if (num_seqs == 0) return ap ? launch_append_only(*ap, static_cast<cudaStream_t>(stream)) : pkv::ok();
  if (!q || !k_pool || !v_pool || !block_tables || !seq_lens || !workspace || !out)
    return fail(PKV_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return fail(PKV_ERR_INVALID_ARG, "%s: q, pools and out must be 16-byte aligned", fn);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  const int64_t max_tokens = int64_t(max_blocks_per_seq) * block_size;
  if (max_tokens > (int64_t(1) << 30)) return fail(PKV_ERR_INVALID_ARG, "%s: max_blocks_per_seq too large", fn);
  if (int64_t(num_blocks) * num_kv_heads * block_size > INT32_MAX)
    return fail(PKV_ERR_INVALID_ARG, "%s: pool has more than 2^31 token rows", fn);
  const WsLayout w = ws_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_tokens, pt);
  if (workspace_bytes < w.total)
    return fail(PKV_ERR_INVALID_ARG, "%s: workspace %zu bytes < %zu needed", fn, workspace_bytes, w.total);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  pkv::DecodeParams p{};
  p.q = q;
  set_single_pool(p, k_pool, v_pool, block_tables, num_blocks, max_blocks_per_seq, block_size);
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.partition_tokens = pt;
  p.max_parts = w.max_parts;
  // scores = scale * k_scale * q·codes; output = v_scale * softmax-weighted codes
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * static_cast<double>(k_scale) * 1.4426950408889634);
  p.v_scale = v_scale;
  p.items = reinterpret_cast<const int4*>(ws + w.items);
  p.n_items = reinterpret_cast<const int32_t*>(ws);
  p.part_m = reinterpret_cast<float*>(ws + w.m);
  p.part_l = reinterpret_cast<float*>(ws + w.l);
  p.part_o = reinterpret_cast<float*>(ws + w.o);
  p.out = out;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t mt = static_cast<int32_t>(max_tokens);
  switch (group) {
    case 1: return launch_decode_tc8<1>(p, seq_lens, num_seqs, mt, ap, s);
    case 2: return launch_decode_tc8<2>(p, seq_lens, num_seqs, mt, ap, s);
    case 4: return launch_decode_tc8<4>(p, seq_lens, num_seqs, mt, ap, s);
    default: return launch_decode_tc8<8>(p, seq_lens, num_seqs, mt, ap, s);
  }
}

}  // namespace

extern "C" int pkv_paged_attention_decode_fp8(const void* q, const void* k_pool, const void* v_pool,
                                              const int32_t* block_tables, const int32_t* seq_lens, int32_t num_seqs,
                                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                              int32_t num_blocks, int32_t max_blocks_per_seq, int32_t block_size,
                                              float scale, float k_scale, float v_scale, int32_t partition_tokens,
                                              void* workspace, size_t workspace_bytes, float* out, void* stream) {
  NvtxRange nvtx_range("pkv_paged_attention_decode_fp8");
  return decode_fp8("pkv_paged_attention_decode_fp8", q, k_pool, v_pool, block_tables, seq_lens, num_seqs,
                    num_q_heads, num_kv_heads, head_dim, num_blocks, max_blocks_per_seq, block_size, scale, k_scale,
                    v_scale, partition_tokens, workspace, workspace_bytes, out, nullptr, stream);
}

extern "C" int pkv_append_and_decode_fp8(const void* k_new, const void* v_new, int32_t src_dtype,
                                         const int32_t* slot_mapping, int32_t n_tokens, const void* q, void* k_pool,
                                         void* v_pool, const int32_t* block_tables, const int32_t* seq_lens,
                                         int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                         int32_t head_dim, int32_t num_blocks, int32_t max_blocks_per_seq,
                                         int32_t block_size, float scale, float k_scale, float v_scale,
                                         int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                                         float* out, void* stream) {
  NvtxRange nvtx_range("pkv_append_and_decode_fp8");
  const char* fn = "pkv_append_and_decode_fp8";
  int rc = check_common(num_kv_heads, head_dim, block_size, src_dtype, fn);
  if (rc) return rc;
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return fail(PKV_ERR_INVALID_ARG, "%s: scales must be positive and finite", fn);
  if (n_tokens < 0 || num_blocks <= 0) return fail(PKV_ERR_INVALID_ARG, "%s: n_tokens/num_blocks", fn);
  if (n_tokens > 0) {
    if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool) return fail(PKV_ERR_INVALID_ARG, "%s: NULL pointer", fn);
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
      return fail(PKV_ERR_INVALID_ARG, "%s: buffers must be 16-byte aligned", fn);
  }
  const float k_inv = static_cast<float>(1.0 / static_cast<double>(k_scale));
  const float v_inv = static_cast<float>(1.0 / static_cast<double>(v_scale));
  PendingAppend ap{single_append(k_new, v_new, slot_mapping, int64_t(n_tokens) * num_kv_heads * (head_dim / 8),
                                 k_pool, v_pool, num_blocks, num_kv_heads, head_dim / 8, block_size, k_inv, v_inv),
                   src_dtype};
  return decode_fp8(fn, q, k_pool, v_pool, block_tables, seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                    num_blocks, max_blocks_per_seq, block_size, scale, k_scale, v_scale, partition_tokens, workspace,
                    workspace_bytes, out, n_tokens > 0 ? &ap : nullptr, stream);
}

// ===========================================================================
// Decode without caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// serving runtimes that reserve nearly all of HBM for their KV pool up front
// (a later cudaMalloc can fail or fragment that reservation), framework
// plugins whose host owns every allocation and forbids direct cudaMalloc, and
// hot loops that must not pay a synchronising cudaMalloc / cudaFree.  For
// them the split-partition scratch lives in this file-scope array instead.
// Every GPU that loads the library holds it (kStaticWorkspaceBytes) until the
// process exits.
// ===========================================================================
namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(64) << 20;  // 64 MiB
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// Device address of g_static_workspace on the current device, looked up once
// per device (the host-side name is only a stand-in for the device array).
int static_workspace_ptr(void** out) {
  static std::mutex mu;
  static void* ptrs[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev >= kMaxDevices) return fail(PKV_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> g(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return PKV_OK;
}

}  // namespace

extern "C" size_t pkv_static_workspace_bytes(void) { return kStaticWorkspaceBytes; }

extern "C" int pkv_paged_attention_decode_static(const void* q, const void* k_pool, const void* v_pool,
                                                 const int32_t* block_tables, const int32_t* seq_lens,
                                                 int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                                 int32_t head_dim, int32_t num_blocks, int32_t max_blocks_per_seq,
                                                 int32_t block_size, float scale, int32_t dtype,
                                                 int32_t partition_tokens, float* out, void* stream) {
  NvtxRange nvtx_range("pkv_paged_attention_decode_static");
  size_t need = 0;
  int rc = pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, block_size,
                                     partition_tokens, &need);
  if (rc) return rc;
  if (need > kStaticWorkspaceBytes)
    return fail(PKV_ERR_INVALID_ARG,
                "pkv_paged_attention_decode_static: these sizes need %zu bytes of scratch, more than the %zu-byte "
                "static workspace; use pkv_paged_attention_decode with a caller-provided workspace",
                need, kStaticWorkspaceBytes);
  if (num_seqs == 0) return pkv::ok();
  void* ws = nullptr;
  rc = static_workspace_ptr(&ws);
  if (rc) return rc;
  return pkv_paged_attention_decode(q, k_pool, v_pool, block_tables, seq_lens, num_seqs, num_q_heads, num_kv_heads,
                                    head_dim, num_blocks, max_blocks_per_seq, block_size, scale, dtype,
                                    partition_tokens, ws, kStaticWorkspaceBytes, out, stream);
}

// =============================================================================
// Paged prefill attention (tcgen05 tensor cores)
// =============================================================================
namespace {

// q [num_q_tokens, Hq, 128] of 16-bit elements viewed as 4-D: x = 64 elements,
// y = head_dim half (128 bytes apart), z = query head, w = token.  A box of
// 64 x 1 x G x (128 / G) lands as 128 rows (token-major, then head) of 128
// bytes, 128-byte swizzled: the A operand of S = Q · Kᵀ.
int make_prefill_q_map(CUtensorMap* m, const void* q, int dtype, int32_t num_q_tokens, int32_t num_q_heads,
                       int32_t group) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[4] = {64, 2, static_cast<cuuint64_t>(num_q_heads), static_cast<cuuint64_t>(num_q_tokens)};
  const cuuint64_t strides[3] = {128, 256, static_cast<cuuint64_t>(num_q_heads) * 256};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(128 / group)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                   const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled (prefill q) failed (%d)", static_cast<int>(r));
  return PKV_OK;
}

// Pool of 16-bit elements, head_dim 128, viewed as in make_pool_map but with
// a box of one head_dim half: 64 x block_size x 1, so the halves of a chunk's
// blocks land in two separate 128-row slabs.
int make_prefill_pool_map(CUtensorMap* m, const void* pool, int dtype, int64_t rows, int32_t block_size) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), 2};
  const cuuint64_t strides[2] = {256, 128};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(block_size), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                   const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled (prefill pool) failed (%d)", static_cast<int>(r));
  return PKV_OK;
}

// Tile counters of the persistent prefill kernel.  A launch draws its tiles
// from one slot and its last CTA re-arms the slot to zero; successive
// launches take successive slots, so launches that overlap on the GPU (up to
// kPrefillSlots of them) never share one.
constexpr int kPrefillSlots = 64;
__device__ unsigned int g_prefill_tiles[kPrefillSlots][2];

int prefill_counter(unsigned int** out) {
  static std::mutex mu;
  static void* base[kMaxDevices] = {};
  static std::atomic<unsigned> next{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev >= kMaxDevices) return fail(PKV_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  {
    std::lock_guard<std::mutex> g(mu);
    if (!base[dev]) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_prefill_tiles);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(prefill tile counters)");
      base[dev] = ptr;
    }
  }
  const unsigned slot = next.fetch_add(1, std::memory_order_relaxed) % kPrefillSlots;
  *out = static_cast<unsigned int*>(base[dev]) + 2 * slot;
  return PKV_OK;
}

// Bytes of the staged f16 copy of V (bf16 pools): a 256-byte record, then
// [num_seqs][max_blocks][Hkv][block_size][128] f16.
size_t prefill_stage_bytes(int64_t num_seqs, int64_t num_kv_heads, int64_t max_blocks, int64_t block_size) {
  return 256 + round256(size_t(num_seqs * max_blocks * num_kv_heads * block_size) * 128 * sizeof(__half));
}

// One launch of the persistent prefill kernel instance <T, G, kF16P>: one
// CTA per SM, its own tile-counter slot.
template <typename T, int G, bool kF16P>
int launch_prefill_instance(const pkv::PrefillParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                            const CUtensorMap& mv, int dev, cudaStream_t stream) {
  auto kern = pkv::prefill_tc_kernel<T, G, kF16P>;
  static std::atomic<bool> configured[kMaxDevices];
  if (dev >= kMaxDevices || !configured[dev].load(std::memory_order_relaxed)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pkv::pf::kSmemBytes));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill)");
    if (dev < kMaxDevices) configured[dev].store(true, std::memory_order_relaxed);
  }
  const int64_t tiles = int64_t(p.n_tiles) * p.num_seqs * p.num_kv_heads;
  const int64_t grid = std::min<int64_t>(sm_count(dev), tiles);  // persistent: one CTA per SM
  unsigned int* ctr = nullptr;
  int rc = prefill_counter(&ctr);
  if (rc) return rc;
  // programmatically serialised: the kernel waits for its predecessor
  // (griddepcontrol.wait) before reading anything
  const cudaError_t e = launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(pkv::pf::kThreads),
                                   pkv::pf::kSmemBytes, stream, p, mq, mk, mv, ctr);
  if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
  return PKV_OK;
}

template <typename T, int G>
int launch_prefill(const pkv::PrefillParams& p, const void* q, const void* k_pool, const void* v_pool, int dtype,
                   void* v_stage, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  CUtensorMap mq, mk, mv;
  int rc = make_prefill_q_map(&mq, q, dtype, p.num_q_tokens, p.num_q_heads, G);
  if (rc) return rc;
  const int64_t rows = int64_t(p.num_blocks) * p.num_kv_heads * p.block_size;
  rc = make_prefill_pool_map(&mk, k_pool, dtype, rows, p.block_size);
  if (rc) return rc;
  rc = make_prefill_pool_map(&mv, v_pool, dtype, rows, p.block_size);
  if (rc) return rc;
  pkv::PrefillParams pp = p;
  CUtensorMap mvs = mv;
  if (v_stage) {
    // V of every sequence's blocks converted to f16 once, then read by the
    // prefill kernel through its own map (same box shape as the pool's)
    static std::atomic<uint32_t> epoch{0};
    pp.epoch = epoch.fetch_add(1, std::memory_order_relaxed) + 1;
    pp.v_staged = 1;
    pp.v_range = static_cast<const uint32_t*>(v_stage);
    unsigned char* copy = static_cast<unsigned char*>(v_stage) + 256;
    const int64_t srows = int64_t(p.num_seqs) * p.max_blocks * p.num_kv_heads * p.block_size;
    rc = make_prefill_pool_map(&mvs, copy, PKV_F16, srows, p.block_size);
    if (rc) return rc;
    pkv::VStageArgs a{};
    a.block_tables = p.block_tables;
    a.seq_lens = p.seq_lens;
    a.v_pool = static_cast<const uint4*>(v_pool);
    a.staged = reinterpret_cast<uint4*>(copy);
    a.range = static_cast<uint32_t*>(v_stage);
    a.epoch = pp.epoch;
    a.num_seqs = p.num_seqs;
    a.num_blocks = p.num_blocks;
    a.max_blocks = p.max_blocks;
    a.block_size = p.block_size;
    a.block_pieces = p.num_kv_heads * p.block_size * 128 / 8;
    // at most two whole blocks per CTA: the CTAs past a sequence's last block
    // return at once and the block scheduler balances sequences of different
    // lengths (a fixed ~8 CTAs per SM over the batch left the CTAs of the
    // longest sequences copying four blocks while the rest had finished)
    const int ny = std::min(p.num_seqs, 65535);
    const int nx = std::max(1, (p.max_blocks + 1) / 2);
    const cudaError_t es = launch_pdl(pkv::stage_v_f16_kernel, dim3(nx, ny), dim3(256), 0, stream, a);
    if (es != cudaSuccess) return cuda_fail(es, "V staging launch");
  }
  // every launch programmatically serialised: each kernel waits for its
  // predecessor (griddepcontrol.wait) before reading anything
  if constexpr (std::is_same<T, __half>::value) {
    rc = launch_prefill_instance<__half, G, true>(pp, mq, mk, mv, dev, stream);
  } else if (v_stage) {
    // the bf16 instance runs only if the staging found a value beyond the
    // f16 range, the f16 one only if it did not; the other returns at once
    rc = launch_prefill_instance<__nv_bfloat16, G, false>(pp, mq, mk, mv, dev, stream);
    if (!rc) rc = launch_prefill_instance<__nv_bfloat16, G, true>(pp, mq, mk, mvs, dev, stream);
  } else {
    rc = launch_prefill_instance<__nv_bfloat16, G, false>(pp, mq, mk, mv, dev, stream);
  }
  if (rc) return rc;
  return pkv::ok();
}

template <typename T>
int dispatch_prefill(int32_t group, const pkv::PrefillParams& p, const void* q, const void* k_pool, const void* v_pool,
                     int dtype, void* v_stage, cudaStream_t s) {
  if (group == 1) return launch_prefill<T, 1>(p, q, k_pool, v_pool, dtype, v_stage, s);
  if (group == 2) return launch_prefill<T, 2>(p, q, k_pool, v_pool, dtype, v_stage, s);
  if (group == 4) return launch_prefill<T, 4>(p, q, k_pool, v_pool, dtype, v_stage, s);
  return launch_prefill<T, 8>(p, q, k_pool, v_pool, dtype, v_stage, s);
}

}  // namespace

extern "C" int pkv_prefill_workspace_size(int32_t num_seqs, int32_t num_kv_heads, int32_t head_dim,
                                          int32_t max_blocks_per_seq, int32_t block_size, int32_t dtype,
                                          size_t* bytes) {
  if (!bytes) return fail(PKV_ERR_INVALID_ARG, "pkv_prefill_workspace_size: bytes is NULL");
  if (num_seqs < 0 || num_kv_heads <= 0 || head_dim <= 0 || max_blocks_per_seq < 0 || block_size <= 0)
    return fail(PKV_ERR_INVALID_ARG, "pkv_prefill_workspace_size: bad sizes");
  *bytes = dtype == PKV_BF16 ? prefill_stage_bytes(num_seqs, num_kv_heads, max_blocks_per_seq, block_size) : 0;
  return pkv::ok();
}

extern "C" int pkv_paged_attention_prefill(const void* q, const void* k_pool, const void* v_pool,
                                           const int32_t* block_tables, const int32_t* seq_lens,
                                           const int32_t* q_start, int32_t num_seqs, int32_t num_q_tokens,
                                           int32_t max_q_len, int32_t num_q_heads, int32_t num_kv_heads,
                                           int32_t head_dim, int32_t num_blocks, int32_t max_blocks_per_seq,
                                           int32_t block_size, float scale, int32_t dtype, void* workspace,
                                           size_t workspace_bytes, float* out, void* stream) {
  NvtxRange nvtx_range("pkv_paged_attention_prefill");
  const char* fn = "pkv_paged_attention_prefill";
  if (dtype != PKV_BF16 && dtype != PKV_F16)
    return fail(PKV_ERR_UNSUPPORTED, "%s: dtype %d not supported (bf16 or f16)", fn, dtype);
  int rc = check_common(num_kv_heads, head_dim, block_size, dtype, fn);
  if (rc) return rc;
  if (head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "%s: head_dim %d not supported (128)", fn, head_dim);
  if (num_seqs < 0 || num_q_tokens < 0 || max_q_len < 0 || num_q_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq < 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad sizes", fn);
  if (num_q_heads % num_kv_heads != 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: num_q_heads %d not a multiple of num_kv_heads %d", fn, num_q_heads,
                num_kv_heads);
  const int32_t group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PKV_ERR_UNSUPPORTED, "%s: group size %d not supported (1, 2, 4 or 8)", fn, group);
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(PKV_ERR_INVALID_ARG, "%s: scale must be positive and finite", fn);
  if (num_seqs == 0 || num_q_tokens == 0 || max_q_len == 0) return pkv::ok();
  if (!q || !k_pool || !v_pool || !block_tables || !seq_lens || !q_start || !out)
    return fail(PKV_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return fail(PKV_ERR_INVALID_ARG, "%s: q, pools and out must be 16-byte aligned", fn);
  if (int64_t(num_blocks) * num_kv_heads * block_size >= (int64_t(1) << 31))
    return fail(PKV_ERR_INVALID_ARG, "%s: pool rows exceed 2^31", fn);
  if (int64_t(max_blocks_per_seq) * block_size >= (int64_t(1) << 31))
    return fail(PKV_ERR_INVALID_ARG, "%s: max_blocks_per_seq * block_size exceeds 2^31", fn);
  const int32_t qt = pkv::pf::kTileRows / group;  // query tokens per tile
  const int64_t n_tiles = (int64_t(max_q_len) + qt - 1) / qt;
  const int64_t grid = n_tiles * num_seqs * num_kv_heads;
  if (grid >= (int64_t(1) << 31)) return fail(PKV_ERR_INVALID_ARG, "%s: too many tiles (%lld)", fn, (long long)grid);
  pkv::PrefillParams p{};
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.q_start = q_start;
  p.out = out;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.num_blocks = num_blocks;
  p.max_blocks = max_blocks_per_seq;
  p.block_size = block_size;
  p.num_q_tokens = num_q_tokens;
  p.max_q_len = max_q_len;
  p.n_tiles = static_cast<int32_t>(n_tiles);
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.stall_cta = g_stall_prefill_cta.load(std::memory_order_relaxed);
  void* v_stage = nullptr;
  if (dtype == PKV_BF16 && workspace) {
    const size_t need = prefill_stage_bytes(num_seqs, num_kv_heads, max_blocks_per_seq, block_size);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(PKV_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
    if (workspace_bytes < need)
      return fail(PKV_ERR_INVALID_ARG, "%s: workspace %zu bytes < %zu needed", fn, workspace_bytes, need);
    if (int64_t(num_seqs) * max_blocks_per_seq * num_kv_heads * block_size >= (int64_t(1) << 31))
      return fail(PKV_ERR_INVALID_ARG, "%s: staged V rows exceed 2^31", fn);
    v_stage = workspace;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == PKV_BF16) return dispatch_prefill<__nv_bfloat16>(group, p, q, k_pool, v_pool, dtype, v_stage, s);
  return dispatch_prefill<__half>(group, p, q, k_pool, v_pool, dtype, nullptr, s);
}

// =============================================================================
// A whole decode step from host buffers
// =============================================================================
extern "C" size_t pkv_step_meta_bytes(int32_t n, int32_t max_blocks_per_seq) {
  if (n <= 0 || max_blocks_per_seq < 0) return 0;
  return size_t(n) * (4 + size_t(max_blocks_per_seq)) * sizeof(int32_t);
}

extern "C" int pkv_decode_step_host(pkv_alloc_t* a, const int64_t* seq_ids, int32_t n, const pkv_step_buffers_t* buf,
                                    void* k_pool, void* v_pool, int32_t num_blocks, int32_t num_q_heads,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                    int32_t max_blocks_per_seq, float scale, int32_t dtype, float k_scale,
                                    float v_scale, int32_t partition_tokens, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("pkv_decode_step_host");
  const char* fn = "pkv_decode_step_host";
  if (!a || !buf || n < 0 || max_blocks_per_seq <= 0 || num_kv_heads <= 0 || num_q_heads <= 0 || head_dim <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad arguments", fn);
  if (n == 0) return pkv::ok();
  if (!seq_ids || !buf->meta_host || !buf->meta_dev || !buf->q_host || !buf->k_host || !buf->v_host ||
      !buf->q_dev || !buf->k_dev || !buf->v_dev || !buf->out_dev)
    return fail(PKV_ERR_INVALID_ARG, "%s: NULL buffer", fn);
  if ((buf->h2d_stream && (!buf->done_event || !buf->compute_done)) ||
      (buf->d2h_stream && (!buf->compute_done || !buf->d2h_done)))
    return fail(PKV_ERR_INVALID_ARG, "%s: a copy stream needs its events", fn);
  const bool fp8 = dtype == PKV_FP8_E4M3;
  if (!fp8 && dtype != PKV_F32 && dtype != PKV_BF16 && dtype != PKV_F16)
    return fail(PKV_ERR_UNSUPPORTED, "%s: dtype %d not supported", fn, dtype);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (buf->wait_event) {
    e = cudaEventSynchronize(static_cast<cudaEvent_t>(buf->wait_event));
    if (e != cudaSuccess) return cuda_fail(e, "pkv_decode_step_host: cudaEventSynchronize");
  }
  int32_t* m = static_cast<int32_t*>(buf->meta_host);
  int32_t* slots = m;
  int32_t* lens = m + n;
  int32_t* cow = m + 2 * n;
  int32_t* tables = m + 4 * n;
  int32_t ncow = 0;
  int rc = pkv_seq_append_slots(a, seq_ids, n, slots, cow, n, &ncow);
  if (rc) return rc;
  rc = pkv_block_tables(a, seq_ids, n, max_blocks_per_seq, tables, lens);
  if (rc) return rc;
  const size_t io = fp8 ? 2 : elem_size(dtype);  // bytes per element of q and of the new rows
  const size_t qb = size_t(n) * num_q_heads * head_dim * io, kb = size_t(n) * num_kv_heads * head_dim * io;
  cudaStream_t hs = buf->h2d_stream ? static_cast<cudaStream_t>(buf->h2d_stream) : s;
  cudaEvent_t compute_done = static_cast<cudaEvent_t>(buf->compute_done);
  e = cudaSuccess;
  if (buf->h2d_stream) e = cudaStreamWaitEvent(hs, compute_done, 0);  // the device buffers' last readers are done
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(buf->meta_dev, buf->meta_host, pkv_step_meta_bytes(n, max_blocks_per_seq),
                        cudaMemcpyHostToDevice, hs);
  if (e == cudaSuccess) e = cudaMemcpyAsync(buf->q_dev, buf->q_host, qb, cudaMemcpyHostToDevice, hs);
  if (e == cudaSuccess) e = cudaMemcpyAsync(buf->k_dev, buf->k_host, kb, cudaMemcpyHostToDevice, hs);
  if (e == cudaSuccess) e = cudaMemcpyAsync(buf->v_dev, buf->v_host, kb, cudaMemcpyHostToDevice, hs);
  if (e == cudaSuccess && buf->done_event) e = cudaEventRecord(static_cast<cudaEvent_t>(buf->done_event), hs);
  if (e == cudaSuccess && buf->h2d_stream) e = cudaStreamWaitEvent(s, static_cast<cudaEvent_t>(buf->done_event), 0);
  if (e == cudaSuccess && buf->d2h_stream) e = cudaStreamWaitEvent(s, static_cast<cudaEvent_t>(buf->d2h_done), 0);
  if (e != cudaSuccess) return cuda_fail(e, "pkv_decode_step_host: host-to-device copies");
  const int32_t* md = static_cast<const int32_t*>(buf->meta_dev);
  if (ncow) {
    rc = pkv_copy_blocks(k_pool, v_pool, md + 2 * n, ncow, num_blocks, num_kv_heads, head_dim, block_size, dtype,
                         stream);
    if (rc) return rc;
  }
  if (fp8) {
    rc = pkv_append_and_decode_fp8(buf->k_dev, buf->v_dev, PKV_F16, md, n, buf->q_dev, k_pool, v_pool, md + 4 * n,
                                   md + n, n, num_q_heads, num_kv_heads, head_dim, num_blocks, max_blocks_per_seq,
                                   block_size, scale, k_scale, v_scale, partition_tokens, workspace, workspace_bytes,
                                   buf->out_dev, stream);
  } else {
    rc = pkv_append_and_decode(buf->k_dev, buf->v_dev, md, n, buf->q_dev, k_pool, v_pool, md + 4 * n, md + n, n,
                               num_q_heads, num_kv_heads, head_dim, num_blocks, max_blocks_per_seq, block_size, scale,
                               dtype, partition_tokens, workspace, workspace_bytes, buf->out_dev, stream);
  }
  if (rc) return rc;
  if (buf->h2d_stream || buf->d2h_stream) {
    e = cudaEventRecord(compute_done, s);
    if (e != cudaSuccess) return cuda_fail(e, "pkv_decode_step_host: cudaEventRecord");
  }
  if (buf->out_host) {
    cudaStream_t ds = buf->d2h_stream ? static_cast<cudaStream_t>(buf->d2h_stream) : s;
    e = buf->d2h_stream ? cudaStreamWaitEvent(ds, compute_done, 0) : cudaSuccess;
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(buf->out_host, buf->out_dev, size_t(n) * num_q_heads * head_dim * sizeof(float),
                          cudaMemcpyDeviceToHost, ds);
    if (e == cudaSuccess && buf->d2h_stream) e = cudaEventRecord(static_cast<cudaEvent_t>(buf->d2h_done), ds);
    if (e != cudaSuccess) return cuda_fail(e, "pkv_decode_step_host: device-to-host copy");
  }
  return pkv::ok();
}
