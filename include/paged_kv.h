/*
 * paged_kv.h — C ABI of libpagedkv: a paged KV cache and PagedAttention decode
 * for NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources cited by page title and section):
 *
 *  - "vLLM's 'memory paging' — PagedAttention illustrated", §2: the KV cache is
 *    cut into fixed-size pages (blocks of 8/16/... tokens); every sequence
 *    keeps a page table of physical blocks that need not be contiguous; a
 *    scheduler hands blocks out from a free list and takes them back.
 *  - same page, §3 phase 1: a new token goes into the sequence's current
 *    block; when that block is full the next token takes a fresh block from
 *    the free list and the table grows by one entry (no copy of old data).
 *  - same page, §3 phase 2: attention reads the table, treats the scattered
 *    blocks as one logically contiguous K and V, and runs ordinary attention
 *    (scores q·Kᵀ, softmax, weighted sum of V).
 *  - same page, §3 phase 3 and §4: blocks shared by several sequences carry a
 *    reference count and are freed by the last sharer; writing into a shared
 *    block goes to a private copy first; admission refuses work that does not
 *    fit instead of running out of memory; abort frees a request's blocks.
 *  - "LLM inference optimisation: principles overview", §3.3: page layout and
 *    block sizes 8/16/32.
 *
 * Conventions
 *  - Every function returns an int status: PKV_OK (0) or a negative PKV_ERR_*.
 *    pkv_last_error_string() gives the text of the calling thread's last error.
 *  - Argument errors are reported synchronously, before anything is launched.
 *  - Device pointers are owned by the caller (allocated e.g. by PyTorch); the
 *    library never allocates or frees device memory at run time (the one fixed
 *    exception is the static scratch of pkv_paged_attention_decode_static,
 *    held from library load to process exit).  Device buffers must be 16-byte
 *    aligned and densely packed in the layouts stated below.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Kernels are launched asynchronously on it; returning PKV_OK means the
 *    launch was accepted.  Faults found by the kernels themselves (a block id
 *    outside the pool, a wait that ran out) are recorded in a device status
 *    word read with pkv_device_status().
 *  - dtype: PKV_F32, PKV_BF16 or PKV_F16 — the element type of q, the new K/V
 *    rows and the K/V pools.  Attention output is always float32.
 *
 * KV pool layout: K and V are separate pools, each
 *     [num_blocks][num_kv_heads][block_size][head_dim]   (head_dim fastest)
 * so one (block, kv head) is a contiguous block_size*head_dim tile.  Slot
 * s = block*block_size + offset names token row `offset` of physical block
 * `block`.  Supported: head_dim in {64, 128}, block_size in {8, 16, 32},
 * num_q_heads / num_kv_heads in {1, 2, 4, 8}.
 */
#ifndef PAGED_KV_H
#define PAGED_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum pkv_status {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = -1,    /* bad size, null pointer, misalignment */
  PKV_ERR_OUT_OF_BLOCKS = -2,  /* not enough free blocks; nothing changed */
  PKV_ERR_UNKNOWN_SEQ = -3,    /* sequence id not present */
  PKV_ERR_UNSUPPORTED = -4,    /* dtype / head_dim / block_size / group size */
  PKV_ERR_CUDA = -5,           /* a CUDA runtime call failed */
  PKV_ERR_DEVICE_TIMEOUT = -6, /* a bounded device wait gave up */
  PKV_ERR_SEQ_EXISTS = -7,     /* sequence id already present */
  PKV_ERR_BAD_BLOCK = -8       /* a kernel met a block id / slot outside the pool */
};

enum pkv_dtype { PKV_F32 = 0, PKV_BF16 = 1, PKV_F16 = 2, PKV_FP8_E4M3 = 3 };

/* Text of the calling thread's most recent error ("" if none).  The pointer
 * stays valid until the thread's next library call. */
const char* pkv_last_error_string(void);

/* Library version string, e.g. "1.0.0". */
const char* pkv_version(void);

/* ------------------------------------------------------------------------ */
/* Host block allocator (vLLM paging page §2, §3 phases 1 and 3, §4).       */
/* All of it runs on the host in integers.  A pkv_alloc_t is not thread-safe:
 * one thread at a time.  Every failing call leaves the allocator unchanged. */
/* ------------------------------------------------------------------------ */

typedef struct pkv_alloc pkv_alloc_t;

typedef struct pkv_stats {
  int64_t num_blocks;
  int64_t block_size;
  int64_t free_blocks;
  int64_t used_blocks;    /* num_blocks - free_blocks */
  int64_t num_seqs;
  int64_t cow_copies;     /* copy-on-write pairs issued since creation */
  int64_t logical_tokens; /* sum of sequence lengths (shared tokens counted per sharer) */
  int64_t waste_tokens;   /* over distinct used blocks: block_size - the fullest sharer's fill */
  int64_t cached_blocks;  /* blocks indexed by the prefix cache (in use or cached-free) */
  int64_t cache_queries;  /* full prompt blocks looked up by pkv_seq_add_cached */
  int64_t cache_hits;     /* of those, blocks reused */
} pkv_stats_t;

/* Create an allocator over blocks 0..num_blocks-1.  The free list is a LIFO
 * stack; `free_order` (num_blocks distinct ids, may be NULL for 0,1,2,...)
 * gives the order in which blocks are first handed out: free_order[0] first.
 * Callers pass a seeded permutation to scatter sequences across the pool.
 * Errors: INVALID_ARG (sizes <= 0, free_order not a permutation). */
int pkv_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* free_order,
                     pkv_alloc_t** out);

/* Free the allocator (NULL is ignored). */
void pkv_alloc_destroy(pkv_alloc_t* a);

/* Admit a sequence that already holds n_tokens tokens (e.g. a prompt):
 * reserves ceil(n_tokens / block_size) blocks at once, or none
 * (admission control, vLLM paging page §4).
 * Errors: SEQ_EXISTS, OUT_OF_BLOCKS, INVALID_ARG (n_tokens < 0). */
int pkv_seq_add(pkv_alloc_t* a, int64_t seq_id, int32_t n_tokens);

/* Admit a sequence whose n_tokens prompt token ids are known, reusing cached
 * blocks of an identical prefix (prefix caching: vLLM paging page §3 phase 3
 * and §5 "enable_prefix_caching"; vLLM production page §5).  Each full block
 * of the prompt is identified by the token ids of the whole prefix through
 * it (64-bit FNV-1a chain hash, verified against stored tokens on every
 * hit).  The longest run of leading full blocks found in the cache is reused
 * (refcount + 1); the rest, including a partial last block, are fresh, and
 * fresh full blocks are registered.  A registered block whose refcount
 * reaches zero stays cached ("cached-free", still counted as free) until a
 * hit revives it or the free stack runs dry and it is evicted, least
 * recently freed first.  *n_cached_tokens (may be NULL) receives the number
 * of leading tokens whose K/V are already in the pool (reused blocks x
 * block_size); the caller computes and appends the rest.  All-or-nothing.
 * Errors: SEQ_EXISTS, OUT_OF_BLOCKS, INVALID_ARG. */
int pkv_seq_add_cached(pkv_alloc_t* a, int64_t seq_id, const int32_t* tokens, int32_t n_tokens,
                       int32_t* n_cached_tokens);

/* Make `child` share every block of `parent` (refcount + 1 each); child gets
 * parent's length.  Prefix sharing, vLLM paging page §3 phase 3.
 * Errors: UNKNOWN_SEQ (parent), SEQ_EXISTS (child). */
int pkv_seq_fork(pkv_alloc_t* a, int64_t parent, int64_t child);

/* Reserve the slot of one new token for each listed sequence, in list order
 * (vLLM paging page §3 phase 1).  For a sequence of length L the new token is
 * position L:
 *   - if L % block_size == 0 a block is popped from the free list (or a
 *     cached-free block is evicted when the list is empty) and appended to
 *     its table;
 *   - else if its last block is shared (refcount > 1) a block is popped, the
 *     pair (old, new) is written to cow_pairs_out (copy the old block's K/V
 *     into the new one before writing the token: pkv_copy_blocks), the old
 *     block's refcount drops by one and the table entry now names the new one;
 *   - the slot table[L / block_size] * block_size + L % block_size is written
 *     to slot_out[i] and the length becomes L + 1.
 * slot_out: int32[n].  cow_pairs_out: int32[cow_capacity][2] (src, dst);
 * *n_cow receives the number of pairs.  At most n pairs are produced, so
 * cow_capacity >= n always suffices.
 * All-or-nothing: on OUT_OF_BLOCKS, UNKNOWN_SEQ or INVALID_ARG (cow_capacity
 * too small) no sequence changes. */
int pkv_seq_append_slots(pkv_alloc_t* a, const int64_t* seq_ids, int32_t n,
                         int32_t* slot_out, int32_t* cow_pairs_out, int32_t cow_capacity,
                         int32_t* n_cow);

/* End (or abort) a sequence: each of its blocks loses one reference, and a
 * block reaching zero goes back on the free stack, in table order (vLLM paging
 * page §3 phase 3, §4 abort).  Errors: UNKNOWN_SEQ. */
int pkv_seq_free(pkv_alloc_t* a, int64_t seq_id);

/* Current length (tokens) of a sequence.  Errors: UNKNOWN_SEQ. */
int pkv_seq_len(const pkv_alloc_t* a, int64_t seq_id, int32_t* len);

/* Write the block tables of the listed sequences as rows of
 * tables_out[n][max_blocks] (unused entries = -1) and their lengths to
 * seq_lens_out[n] (may be NULL).  Errors: UNKNOWN_SEQ, INVALID_ARG (a table
 * longer than max_blocks). */
int pkv_block_tables(const pkv_alloc_t* a, const int64_t* seq_ids, int32_t n, int32_t max_blocks,
                     int32_t* tables_out, int32_t* seq_lens_out);

/* Usage counters (vLLM paging page §5 lists KV cache usage as the metric to
 * watch).  Errors: INVALID_ARG. */
int pkv_alloc_stats(const pkv_alloc_t* a, pkv_stats_t* out);

/* ------------------------------------------------------------------------ */
/* Device operations (sm_100a).                                             */
/* ------------------------------------------------------------------------ */

/* KV append ("reshape_and_cache"): for each i < n_tokens with
 * slot_mapping[i] >= 0, copy rows k_new[i][h][:] and v_new[i][h][:] (all
 * heads) into slot slot_mapping[i] of k_pool / v_pool; slot < 0 is a padding
 * token and writes nothing.  Bit-exact copy (vLLM paging page §3 phase 1;
 * optimisation-overview page §2.2: O(1) append, no copy of old data).
 * k_new, v_new: dtype[n_tokens][num_kv_heads][head_dim]; slot_mapping:
 * int32[n_tokens] on the device.  A slot >= num_blocks*block_size is skipped
 * and recorded as PKV_ERR_BAD_BLOCK in the device status.
 * Two tokens given the same slot: which write wins is unspecified. */
int pkv_kv_append(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                  int32_t n_tokens, void* k_pool, void* v_pool, int32_t num_blocks,
                  int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t dtype,
                  void* stream);

/* Copy whole blocks (every head and offset of K and V) src -> dst for each
 * pair in block_pairs: int32[n_pairs][2] on the device — the copy-on-write
 * step of the vLLM paging page §3 phase 3.  dtype may also be PKV_FP8_E4M3.  Pairs must not chain (no dst is
 * another pair's src) and dsts must be distinct; pairs from
 * pkv_seq_append_slots satisfy both.  Ids outside the pool are skipped and
 * recorded as PKV_ERR_BAD_BLOCK. */
int pkv_copy_blocks(void* k_pool, void* v_pool, const int32_t* block_pairs, int32_t n_pairs,
                    int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim,
                    int32_t block_size, int32_t dtype, void* stream);

/* Bytes of device workspace pkv_paged_attention_decode needs for these sizes
 * (split-partition partials and the work list).  partition_tokens as for the
 * decode call (0 = automatic); the value depends only on the arguments. */
int pkv_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t max_blocks_per_seq, int32_t block_size,
                              int32_t partition_tokens, size_t* bytes);

/* PagedAttention decode (vLLM paging page §3 phase 2): for every sequence b
 * and query head h, with G = num_q_heads / num_kv_heads and g = h / G,
 *     out[b][h][:] = sum_t softmax_t(scale * q[b][h]·K_b[t][g]) * V_b[t][g][:]
 * over the seq_lens[b] tokens t of sequence b, where token t of b lives in
 * physical block block_tables[b][t / block_size] at offset t % block_size.
 * No mask: the decode query is the newest position and sees every cached
 * token (call pkv_kv_append first to include the new token itself).
 * seq_lens[b] == 0 gives zeros.
 *
 * q: dtype[num_seqs][num_q_heads][head_dim]; block_tables:
 * int32[num_seqs][max_blocks_per_seq]; seq_lens: int32[num_seqs], each in
 * [0, max_blocks_per_seq*block_size]; out: float32[num_seqs][num_q_heads][head_dim].
 * The softmax is single-pass (online max and sum, fp32 accumulation).
 * Sequences longer than partition_tokens are split into partitions of that
 * many tokens (a multiple of block_size; 0 = automatic), whose partial
 * results are merged by a second kernel with the max/sum rescaling.
 * workspace: at least pkv_decode_workspace_size(...) bytes of device memory,
 * 256-byte aligned, used as scratch for the duration of the call (do not
 * share one workspace between calls that may run concurrently).
 * Table entries outside [0, num_blocks) are not read; they are recorded as
 * PKV_ERR_BAD_BLOCK and block 0 is read in their place. */
int pkv_paged_attention_decode(const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, const int32_t* seq_lens,
                               int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t num_blocks, int32_t max_blocks_per_seq,
                               int32_t block_size, float scale, int32_t dtype,
                               int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                               float* out, void* stream);

/* KV append and decode of one step in one call: the result of
 * pkv_kv_append(k_new, v_new, slot_mapping, n_tokens, ...) followed by
 * pkv_paged_attention_decode(q, ...) on the same stream, every argument
 * meaning what it means there (vLLM paging page §3, phases 1 and 2 of a
 * decode step).  The new rows are written by the launch that builds the
 * decode work list, so a step pays for one launch fewer; the decode kernel
 * starts reading only after that launch has finished.  Pool contents and
 * outputs are bit-identical to the two-call form.  n_tokens = 0 skips the
 * append; num_seqs = 0 skips the decode.  Every argument is checked before
 * anything is launched; errors as for the two calls.  Copy-on-write pairs of
 * the step (pkv_copy_blocks) must be copied before this call. */
int pkv_append_and_decode(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                          int32_t n_tokens, const void* q, void* k_pool, void* v_pool,
                          const int32_t* block_tables, const int32_t* seq_lens, int32_t num_seqs,
                          int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t num_blocks, int32_t max_blocks_per_seq, int32_t block_size,
                          float scale, int32_t dtype, int32_t partition_tokens, void* workspace,
                          size_t workspace_bytes, float* out, void* stream);

/* One whole decode step from host buffers in a single call (vLLM paging page
 * §3: phase 1 reservation, phase 3 copy-on-write, phase 2 attention), for
 * serving loops that want one crossing of the library boundary per step:
 *   1. wait for buf->wait_event (if not NULL) - the copy that last read
 *      buf->meta_host is done;
 *   2. pkv_seq_append_slots + pkv_block_tables for seq_ids into
 *      buf->meta_host, laid out as int32 slots[n] | seq_lens[n] | cow[2n] |
 *      tables[n][max_blocks_per_seq] (pkv_step_meta_bytes(n, max_blocks));
 *   3. host-to-device copies (cudaMemcpyAsync on `stream`) of that metadata
 *      to buf->meta_dev and of the new rows q_host [n][Hq][D],
 *      k_host / v_host [n][Hkv][D] to q_dev / k_dev / v_dev (element type:
 *      dtype, or float16 for e4m3 pools); then record buf->done_event (if
 *      not NULL);
 *   4. pkv_copy_blocks for the copy-on-write pairs, then
 *      pkv_append_and_decode (or _fp8) into buf->out_dev [n][Hq][D] float32;
 *   5. if buf->out_host is not NULL, copy out_dev to it (device to host).
 * Every host buffer should be pinned for the copies to be asynchronous.
 * k_scale / v_scale are used for e4m3 pools only.
 * Overlap (optional): with h2d_stream set, the host-to-device copies run on
 * it after it waits for compute_done (the previous kernels that read these
 * device buffers), and `stream` waits for done_event before the kernels; with
 * d2h_stream set, `stream` records compute_done after the kernels, the copy
 * back runs on d2h_stream after it, and d2h_done is recorded there (the
 * next use of out_dev waits for it).  Alternating two buffer sets then lets
 * the copies of neighbouring steps run under this step's kernels.   Errors: those of the
 * calls above; argument errors leave the allocator unchanged, but once the
 * slots are reserved (step 2) a later device error leaves them reserved. */
typedef struct pkv_step_buffers {
  void* meta_host;
  void* meta_dev;
  const void* q_host;
  const void* k_host;
  const void* v_host;
  void* q_dev;
  void* k_dev;
  void* v_dev;
  float* out_dev;
  float* out_host;
  void* wait_event;
  void* done_event;
  void* h2d_stream;   /* cudaStream_t or NULL */
  void* d2h_stream;   /* cudaStream_t or NULL */
  void* compute_done; /* cudaEvent_t; needed with either stream */
  void* d2h_done;     /* cudaEvent_t; needed with d2h_stream */
} pkv_step_buffers_t;

size_t pkv_step_meta_bytes(int32_t n, int32_t max_blocks_per_seq);

int pkv_decode_step_host(pkv_alloc_t* a, const int64_t* seq_ids, int32_t n, const pkv_step_buffers_t* buf,
                         void* k_pool, void* v_pool, int32_t num_blocks, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         int32_t max_blocks_per_seq, float scale, int32_t dtype, float k_scale,
                         float v_scale, int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Paged prefill attention (chunked prefill: vLLM production page §2;
 * optimisation-overview page §2.3): sequence b brings
 * n_b = q_start[b+1] - q_start[b] new query rows, stored at rows
 * q_start[b] .. q_start[b+1]-1 of q, whose K/V are already in the pool
 * (written by pkv_kv_append), so the pool holds seq_lens[b] tokens of which
 * the last n_b are the chunk's.  Row i of the chunk sits at position
 * p = seq_lens[b] - n_b + i and attends causally to tokens 0 .. p:
 *     out[q_start[b]+i][h][:] = sum_{t<=p} softmax_t(scale * q·K_b[t][g]) * V_b[t][g][:]
 * with g = h / G, G = num_q_heads / num_kv_heads, tokens reached through the
 * block table as in pkv_paged_attention_decode.  A one-row chunk is a decode
 * query.
 *
 * q: dtype[num_q_tokens][num_q_heads][128]; q_start: int32[num_seqs + 1],
 * non-decreasing, q_start[0] >= 0, q_start[num_seqs] <= num_q_tokens;
 * max_q_len: an upper bound of every n_b (sets the launch grid);
 * block_tables / seq_lens as for decode; out: float32[num_q_tokens][num_q_heads][128]
 * (rows outside every chunk are not written).  dtype PKV_BF16 or PKV_F16,
 * head_dim 128, G in {1, 2, 4, 8}, block_size 8, 16 or 32; others return
 * PKV_ERR_UNSUPPORTED.  q, pools and out 16-byte aligned; scale positive
 * and finite (else PKV_ERR_INVALID_ARG).
 * Computed on the tcgen05 tensor cores with fp32 accumulation.  The
 * softmax weights P enter the P·V product as one f16 value (relative error
 * 2^-11 per weight; the output within about 5e-4 of the output scale) for
 * f16 pools, and for bf16 pools given a workspace: the call then first
 * copies V of every block the batch reaches into the workspace as f16 (exact
 * for bf16 magnitudes in [2^-14, 65504], smaller ones rounded to f16
 * subnormals, absolute error at most 2^-25) and the P·V product reads the
 * copy.  Without a workspace (NULL), or if some V value of the batch lies
 * beyond the f16 range, bf16 pools take two bf16 passes (P as hi + lo
 * halves, within about 1e-5 of the exact softmax) over the pool's own V.
 * workspace: at least pkv_prefill_workspace_size() bytes of device memory,
 * 256-byte aligned, owned by the caller and overwritten by the call (NULL or
 * ignored for f16 pools); calls that overlap on the GPU need their own.  A
 * sequence whose chunk is longer than
 * seq_lens[b] or max_q_len is skipped and recorded as PKV_ERR_INVALID_ARG;
 * table entries outside [0, num_blocks) as PKV_ERR_BAD_BLOCK (block 0 read
 * instead), both in the device status.  The kernel runs one CTA per SM,
 * which draws tiles from a counter inside the library; calls take the
 * library's 64 counters in turn, so up to 64 calls may overlap on the GPU
 * (for instance on different streams). */
int pkv_paged_attention_prefill(const void* q, const void* k_pool, const void* v_pool,
                                const int32_t* block_tables, const int32_t* seq_lens,
                                const int32_t* q_start, int32_t num_seqs, int32_t num_q_tokens,
                                int32_t max_q_len, int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim, int32_t num_blocks, int32_t max_blocks_per_seq,
                                int32_t block_size, float scale, int32_t dtype, void* workspace,
                                size_t workspace_bytes, float* out, void* stream);

/* Bytes of the workspace pkv_paged_attention_prefill takes for a batch of
 * num_seqs sequences with tables of max_blocks_per_seq entries: for bf16
 * pools a 256-byte record plus the f16 copy of V,
 * [num_seqs][max_blocks_per_seq][num_kv_heads][block_size][head_dim]
 * (2 bytes per element); 0 for f16 pools.  Host only, no device access. */
int pkv_prefill_workspace_size(int32_t num_seqs, int32_t num_kv_heads, int32_t head_dim,
                               int32_t max_blocks_per_seq, int32_t block_size, int32_t dtype,
                               size_t* bytes);

/* PagedAttention decode exactly as pkv_paged_attention_decode, for callers
 * that cannot allocate device memory when they decode: serving runtimes that
 * have reserved nearly all of HBM for their KV pool up front, framework
 * plugins whose host owns every allocation, hot loops that must not pay a
 * synchronising cudaMalloc/cudaFree.  (The source pages have no counterpart:
 * this is a library convenience.)  The scratch space comes from a static
 * device array inside the library, pkv_static_workspace_bytes() bytes
 * (64 MiB) on every GPU that loads the library, held until the process exits;
 * this call allocates nothing.
 *  - Sizes whose scratch (pkv_decode_workspace_size) exceeds that limit are
 *    rejected with PKV_ERR_INVALID_ARG before anything is launched.
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress (once per device); make that first call before any
 *    stream capture.
 *  - All calls share the one array, and it keeps the last call's contents
 *    (every value a call reads it writes first, so nothing needs clearing).
 *    Calls that overlap on the GPU (different streams, no ordering between
 *    them) race on it: serialise them, or use pkv_paged_attention_decode with
 *    separate workspaces.
 * Arguments, layouts and results as for pkv_paged_attention_decode. */
int pkv_paged_attention_decode_static(const void* q, const void* k_pool, const void* v_pool,
                                      const int32_t* block_tables, const int32_t* seq_lens, int32_t num_seqs,
                                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t num_blocks, int32_t max_blocks_per_seq, int32_t block_size,
                                      float scale, int32_t dtype, int32_t partition_tokens, float* out,
                                      void* stream);

/* Size in bytes of the static workspace used by
 * pkv_paged_attention_decode_static. */
size_t pkv_static_workspace_bytes(void);

/* ------------------------------------------------------------------------ */
/* FP8 (e4m3) KV cache ("LLM inference optimisation: principles overview"   */
/* §5.1: storing the KV cache as FP8 halves its bytes).                     */
/* Pools hold e4m3 codes (uint8, same [num_blocks][num_kv_heads][block_size] */
/* [head_dim] layout); element value = k_scale * e4m3(code) for K and        */
/* v_scale * e4m3(code) for V (one fp32 scale per pool).  e4m3: 1 sign, 4    */
/* exponent (bias 7), 3 mantissa bits, no infinities, 0x7F/0xFF = NaN,       */
/* largest finite 448.                                                       */
/* ------------------------------------------------------------------------ */

/* Append into e4m3 pools: each element x of the new rows (src_dtype PKV_F32,
 * PKV_BF16 or PKV_F16, layout as pkv_kv_append) is stored as the e4m3 code
 * nearest to x * (1/scale), the product taken in fp32 with the fp32
 * reciprocal of the scale, ties to even, saturating to +-448.  Slots as for
 * pkv_kv_append (slot < 0 skipped, out-of-pool recorded as BAD_BLOCK).
 * Errors: INVALID_ARG (scales not positive/finite, misalignment),
 * UNSUPPORTED (head_dim, block_size, src_dtype). */
int pkv_kv_append_fp8(const void* k_new, const void* v_new, int32_t src_dtype, const int32_t* slot_mapping,
                      int32_t n_tokens, void* k_pool, void* v_pool, int32_t num_blocks, int32_t num_kv_heads,
                      int32_t head_dim, int32_t block_size, float k_scale, float v_scale, void* stream);

/* PagedAttention decode over e4m3 pools: the result of
 * pkv_paged_attention_decode on the dequantised values (scores
 * scale * k_scale * q·code, output v_scale * the softmax-weighted codes).
 * q is float16 [num_seqs][num_q_heads][head_dim]; head_dim must be 128;
 * group sizes 1, 2, 4, 8; partition_tokens a multiple of 16 (0 =
 * automatic).  Workspace as sized by
 * pkv_decode_workspace_size with the same arguments. */
int pkv_paged_attention_decode_fp8(const void* q, const void* k_pool, const void* v_pool,
                                   const int32_t* block_tables, const int32_t* seq_lens, int32_t num_seqs,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                                   int32_t max_blocks_per_seq, int32_t block_size, float scale, float k_scale,
                                   float v_scale, int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                                   float* out, void* stream);

/* One pool of a batch that spans several pools (adaptive block size,
 * "LLM inference optimisation: principles overview" §3.3: pools of 32-, 16-
 * and 8-token blocks for short, medium and long sequences).  The pool's
 * sequences are the next num_seqs rows of the batch, in pool order; row r of
 * block_tables is the pool's r-th sequence.  Layouts as for a single pool. */
typedef struct pkv_pool {
  void* k_pool;                 /* [num_blocks][num_kv_heads][block_size][head_dim] */
  void* v_pool;
  const int32_t* block_tables;  /* [num_seqs][max_blocks_per_seq], physical blocks of this pool */
  int32_t num_blocks;
  int32_t block_size;           /* 8, 16 or 32 */
  int32_t max_blocks_per_seq;
  int32_t num_seqs;             /* may be 0 */
} pkv_pool_t;

/* Workspace bytes of pkv_append_and_decode_pools for these pools (sizes
 * only; the pointers are not read).  Host only. */
int pkv_decode_pools_workspace_size(const pkv_pool_t* pools, int32_t n_pools, int32_t num_q_heads,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t partition_tokens,
                                    size_t* bytes);

/* pkv_append_and_decode over a batch whose sequences live in up to 3 pools of
 * different block sizes, in one launch sequence (append + plan, decode,
 * merge) instead of one call per pool.  Row b of k_new / v_new [N][Hkv][D],
 * slot_mapping [N], q [N][Hq][D], seq_lens [N] and out [N][Hq][D] belongs to
 * pool c for sum_{i<c} num_seqs_i <= b < sum_{i<=c} num_seqs_i (N = the sum
 * over the pools); slot_mapping[b] is a slot of that pool (< 0: nothing
 * written), seq_lens[b] counts its tokens after the append.  Every sequence
 * gets the result pkv_append_and_decode would give on its own pool (equal
 * within rounding: the work of a batch is shared out differently).  dtype
 * PKV_BF16 or PKV_F16, head_dim 128, num_q_heads / num_kv_heads in {2, 4, 8},
 * 1 <= n_pools <= 3, partition_tokens (0 = 512) a multiple of 16 and of
 * every pool's block_size; others return PKV_ERR_UNSUPPORTED or
 * PKV_ERR_INVALID_ARG before any launch.  workspace: at least
 * pkv_decode_pools_workspace_size() bytes, 256-byte aligned. */
int pkv_append_and_decode_pools(const pkv_pool_t* pools, int32_t n_pools, const void* k_new,
                                const void* v_new, const int32_t* slot_mapping, const void* q,
                                const int32_t* seq_lens, int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim, float scale, int32_t dtype, int32_t partition_tokens,
                                void* workspace, size_t workspace_bytes, float* out, void* stream);

/* e4m3 form of pkv_append_and_decode: pkv_kv_append_fp8(k_new, v_new,
 * src_dtype, slot_mapping, n_tokens, ..., k_scale, v_scale) followed by
 * pkv_paged_attention_decode_fp8(q, ...), in one call with the same
 * launches saved and the same guarantees (bit-identical codes and outputs). */
int pkv_append_and_decode_fp8(const void* k_new, const void* v_new, int32_t src_dtype,
                              const int32_t* slot_mapping, int32_t n_tokens, const void* q,
                              void* k_pool, void* v_pool, const int32_t* block_tables,
                              const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                              int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                              int32_t max_blocks_per_seq, int32_t block_size, float scale,
                              float k_scale, float v_scale, int32_t partition_tokens,
                              void* workspace, size_t workspace_bytes, float* out, void* stream);

/* Synchronise `stream`, then read the device status word of the current
 * device into *status: PKV_OK, or the first PKV_ERR_BAD_BLOCK /
 * PKV_ERR_DEVICE_TIMEOUT a kernel recorded since the last clear.  clear != 0
 * resets it to PKV_OK.  Returns PKV_ERR_CUDA if the synchronisation failed. */
int pkv_device_status(void* stream, int32_t* status, int32_t clear);

/* Test support for the decode kernels' bounded waits (no counterpart in the
 * pages; failure detection).  Every wait of a decode consumer for a chunk of
 * K/V gives up after a limit (1 s), records PKV_ERR_DEVICE_TIMEOUT in the
 * status word and lets the CTA finish, so a stalled copy costs an error code
 * instead of a hung GPU.  This call makes that path run on demand: for the
 * decode launches that follow (pkv_paged_attention_decode, _fp8, _static and
 * the append-and-decode forms), the producer of CTA `cta` skips the copies
 * of that CTA's first work unit, so their consumers wait for chunks that
 * never arrive and give up after the limit; the producer still waits, with
 * the same limit, for every copy it did issue before its CTA exits.  cta < 0
 * restores normal operation (the default).  Outputs of a stalled call are
 * unspecified; decode does not write the pools.  Process-wide setting, read
 * at each launch; always returns PKV_OK. */
int pkv_debug_stall_decode(int32_t cta);

/* The same for the prefill kernel (pkv_paged_attention_prefill): every wait
 * of its roles gives up after the same limit (1 s), records
 * PKV_ERR_DEVICE_TIMEOUT and sets the CTA's abort flag, after which every
 * role of the CTA leaves its tile loop.  For the prefill launches that
 * follow, the K producer of CTA `cta` skips its first chunk of K, so the MMA
 * warp waits for a chunk that never arrives and gives up after the limit;
 * the producers still wait, with the same limit, for every copy they did
 * issue before the CTA exits.  The other CTAs finish their tiles.  cta < 0
 * restores normal operation (the default).  Outputs of a stalled call are
 * unspecified; prefill does not write the pools.  Process-wide setting,
 * read at each call; always returns PKV_OK. */
int pkv_debug_stall_prefill(int32_t cta);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_H */
