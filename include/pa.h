/*
 * pa.h -- C ABI of the B200 paged KV-cache decode library (libpa.so).
 *
 * The operation is PagedAttention decode as the pages describe it: each
 * sequence's KV cache lives in fixed-size physical blocks (16 or 32 tokens;
 * "vLLM Architecture, Memory and Benchmarks Deep Dive", section 2), a
 * per-sequence block table maps logical blocks to physical ones so that the
 * paged cache looks contiguous to attention ("Optimizing LLM Inference: A Deep
 * Dive into vLLM's PagedAttention and Continuous Batching", section
 * "PagedAttention: Borrowing a 50-Year-Old OS Masterpiece"), new tokens go into
 * blocks handed out on demand (same page as the first, section 2, "On-Demand
 * Allocation"), and query heads share KV heads (grouped-query attention, same
 * page, section 1).
 *
 * Conventions shared by every call
 *   - Pointers named as device pointers must point to memory of the current
 *     CUDA device; the caller owns all memory.  The library never allocates,
 *     frees or synchronises; each call enqueues its kernels on `stream` (a
 *     cudaStream_t; NULL = the legacy default stream) and returns.
 *   - Tensors are dense and row-major (C order).  Shapes use
 *       B   = num_seqs (one new token per sequence),
 *       Hq  = num_q_heads, Hkv = num_kv_heads (Hq / Hkv in {1, 2, 4, 8}),
 *       d   = head_dim in {64, 128, 256},
 *       bs  = block_size in {4, 8, 16, 32},
 *       nb  = num_blocks (physical blocks in each pool).
 *     K and V pools are [nb, bs, Hkv, d]; token t of sequence b lives in
 *     physical block block_tables[b * max_blocks + t / bs], row t % bs.
 *   - Query head hq attends with KV head hq / (Hq / Hkv).
 *   - context_lens[b] counts every cached token of sequence b including the
 *     one being decoded; a length of 0 gives a zero output.
 *   - Element types: PA_DTYPE_F32 (binary32) or PA_DTYPE_BF16 (bfloat16).
 *     Attention accumulates in fp32 and writes `out` in the input type.
 *   - Base pointers of element arrays must be 16-byte aligned.
 *   - Errors the host can see (null pointer, unsupported shape, workspace too
 *     small) return a status and launch nothing.  Errors only the device can
 *     see never trap: the kernel ORs a PA_DEV_* bit into *dev_status (if
 *     dev_status is not NULL), skips the offending access, and the affected
 *     output is zeros (attention) or left untouched (cache write).
 *   - Inputs and outputs must not overlap.
 *   - Every call is asynchronous on `stream` and keeps stream order.  The
 *     decode and cache-write kernels are launched as programmatic dependents
 *     of the kernel before them on the stream (programmatic dependent
 *     launch), and each lets the kernel after it start early, so that a
 *     kernel's set-up overlaps the tail of the one ahead.  The cache write
 *     touches no memory before the kernel ahead has completed.  The decode
 *     kernels read context_lens, block_tables and the K/V pool rows of
 *     cached tokens other than each sequence's last one before it has
 *     completed (the query, the last rows, the outputs and the workspace
 *     after; the query rows are only prefetched into L2 before, which reads
 *     no value): a kernel ahead of them that allows an early start
 *     (griddepcontrol.launch_dependents) must not write those arrays or
 *     rows.  pa_reshape_and_cache, which stores exactly each sequence's
 *     last row, is such a kernel and is safe; kernels that do not allow an
 *     early start, host copies and this library's other kernels need no
 *     care.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, Hq % Hkv != 0, ... */
    PA_ERR_UNSUPPORTED = 2,  /* head_dim / block_size / group / dtype not built */
    PA_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed */
    PA_ERR_WORKSPACE = 4     /* caller-provided workspace too small */
} pa_status;

typedef enum pa_dtype {
    PA_DTYPE_F32 = 0,
    PA_DTYPE_BF16 = 1,
    PA_DTYPE_FP8_E4M3 = 2   /* pools only: pa_copy_blocks, pa_swap_blocks */
} pa_dtype;

/* Bits a kernel ORs into *dev_status. */
#define PA_DEV_BAD_SLOT 0x1      /* cache write: slot >= nb * bs (row not written) */
#define PA_DEV_BAD_BLOCK 0x2     /* a block-table entry read is outside [0, nb) */
#define PA_DEV_BAD_CONTEXT 0x4   /* context_lens[b] < 0 or > max_blocks * bs */
#define PA_DEV_WAIT_TIMEOUT 0x8  /* a bounded wait for an async copy ran out */

/*
 * pa_reshape_and_cache -- store each new token's K and V into its slot.
 *
 * Source: the new token's KV is kept in the block handed out for it
 * ("vLLM Architecture, Memory and Benchmarks Deep Dive", section 2, "On-Demand
 * Allocation"; section 1 for what the KV cache holds).
 *
 *   key, value    device, [num_tokens, Hkv, d], read only.
 *   k_pool,v_pool device, [nb, bs, Hkv, d]; row (slot / bs, slot % bs) of
 *                 every head is overwritten for each token with slot >= 0.
 *   slot_mapping  device, [num_tokens] int64.  A negative slot means padding:
 *                 the token is skipped.  A slot >= nb * bs sets
 *                 PA_DEV_BAD_SLOT and the token is skipped.
 *   The copy is bit-exact; nothing else in the pools changes.  Two tokens
 *   with the same slot race (one of them wins).
 */
pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_pool, void *v_pool,
                               const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                               int32_t *dev_status, void *stream);

/*
 * pa_decode_attention -- single-query GQA attention over the paged cache.
 *
 *   out[b, hq, :] = sum_t p_t V[t, hq / G, :] / sum_t p_t,
 *   p_t = exp(s_t - max_t s_t),  s_t = scale * q[b, hq, :] . K[t, hq / G, :],
 * over the tokens t < context_lens[b] of sequence b, gathered through its
 * block table (the definition above is exact softmax attention; the library
 * computes it with an online softmax in fp32 over 16-token tiles and, where a
 * sequence's tiles are spread over several warps, merges the pieces by the
 * log-sum-exp rule, as in flash-decoding).
 *
 *   out            device, [B, Hq, d], written.
 *   query          device, [B, Hq, d].
 *   k_pool,v_pool  device, [nb, bs, Hkv, d].
 *   block_tables   device, [B, max_blocks_per_seq] int32; entries at or past
 *                  ceil(context_lens[b] / bs) are never read.
 *   context_lens   device, [B] int32.
 *   max_context_len host hint, >= every context_lens[b]; used to size the
 *                  grid.  Must be <= max_blocks_per_seq * bs.
 *   scale          softmax scale (usually 1 / sqrt(d)).
 *   workspace      device scratch of workspace_bytes bytes (may be NULL / 0).
 *                  With at least pa_decode_workspace_bytes() bytes the work is
 *                  split evenly over the GPU's SMs (each CTA owns an equal
 *                  share of the batch's 16-token tiles, whatever the lengths)
 *                  and the pieces of a sequence that straddles CTAs are
 *                  merged inside the kernel through the workspace; with less,
 *                  every (sequence, group of KV heads) is processed by one
 *                  CTA.  Both are exact to the same tolerance.  Contents need
 *                  no initialisation and are garbage afterwards; calls
 *                  sharing a workspace must not run concurrently.
 *   dev_status     device int32 or NULL (see PA_DEV_*).
 */
pa_status pa_decode_attention(void *out, const void *query, const void *k_pool,
                              const void *v_pool, const int32_t *block_tables,
                              int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                              int max_context_len, int num_q_heads, int num_kv_heads,
                              int head_dim, int block_size, int64_t num_blocks, float scale,
                              pa_dtype dtype, void *workspace, size_t workspace_bytes,
                              int32_t *dev_status, void *stream);

/* Workspace bytes pa_decode_attention wants for these sizes (enough for GPUs
 * of up to 256 SMs; about 8.7 MB for Hkv = 4, Hq/Hkv = 4, d = 256).  Host
 * only; touches no device.  num_seqs and max_context_len are accepted for
 * symmetry and unused. */
size_t pa_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_context_len);

/* ceil(max_context_len / partition_size), at least 1. Host only. */
int pa_num_partitions(int max_context_len, int partition_size);

/* Bytes of the three split-K buffers below for max_partitions partitions:
 * tmp_out B*Hq*P*d floats, max_logits and exp_sums B*Hq*P floats each.
 * Host only. */
size_t pa_splitk_workspace_bytes(int num_seqs, int num_q_heads, int head_dim,
                                 int max_partitions);

/*
 * pa_decode_splitk -- the partition pass of flash-decoding, made explicit.
 *
 * Partition p of sequence b covers tokens [p * P, min((p + 1) * P, ctx_b)),
 * P = partition_size (a multiple of 16), for p < n_b = max(1, ceil(ctx_b/P)).
 * For every (b, hq, p < n_b) it writes
 *   max_logits[b, hq, p]      m_p = max logit s_t over the partition,
 *   exp_sums[b, hq, p]        l_p = sum exp(s_t - m_p),
 *   tmp_out[b, hq, p, :]      sum exp(s_t - m_p) V_t / l_p,
 * with logits in natural-log units (s_t = scale * q . k).  An empty
 * partition (ctx_b = 0) gives m = -inf, l = 0, tmp = 0.  Entries with
 * p >= n_b are not touched.  For sequences with n_b == 1 it also writes the
 * final out[b, :, :]; pa_splitk_reduce finishes the others.
 *   max_partitions >= ceil(max_context_len / P); buffers as in
 *   pa_splitk_workspace_bytes, device, fp32.  Other arguments as in
 *   pa_decode_attention.
 */
pa_status pa_decode_splitk(void *out, const void *query, const void *k_pool, const void *v_pool,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int num_seqs, int max_context_len,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int64_t num_blocks, float scale, pa_dtype dtype, int partition_size,
                           int max_partitions, float *tmp_out, float *max_logits,
                           float *exp_sums, int32_t *dev_status, void *stream);

/*
 * pa_splitk_reduce -- merge the partitions of every sequence with n_b > 1:
 *   M = max_p m_p,  w_p = l_p exp(m_p - M),
 *   out[b, hq, :] = sum_p w_p tmp_out[b, hq, p, :] / sum_p w_p.
 * Sequences with n_b == 1 are left alone (pa_decode_splitk wrote them).
 * Arguments as in pa_decode_splitk; out is written in `dtype`.
 */
pa_status pa_splitk_reduce(void *out, const float *tmp_out, const float *max_logits,
                           const float *exp_sums, const int32_t *context_lens, int num_seqs,
                           int num_q_heads, int head_dim, int partition_size,
                           int max_partitions, pa_dtype dtype, void *stream);

/*
 * pa_prefill_attention -- chunked prefill over the paged cache: a chunk of
 * query tokens per sequence attends, causally, to everything the sequence
 * has cached ("vLLM Architecture, Memory and Benchmarks Deep Dive",
 * section 4, "Chunked Prefill": long prompts are cut into chunks, e.g. 512
 * tokens, that run beside decode; section 2: the block table).
 *
 * Sequence b's chunk is query rows cu_q_lens[b] .. cu_q_lens[b + 1] - 1
 * (n_b rows); context_lens[b] counts every cached token including the chunk
 * (whose K/V pa_reshape_and_cache has already written), so chunk row j sits
 * at position ctx_b - n_b + j and attends to the keys at positions 0 .. that
 * position.  Query head hq uses KV head hq / (Hq / Hkv).
 *   out            device, [total_q, Hq, d] bf16, written (rows of every chunk).
 *   query          device, [total_q, Hq, d] bf16.
 *   cu_q_lens      device, [num_seqs + 1] int32, non-decreasing from 0.
 *   max_q_len      host hint, >= every n_b, <= max_context_len.
 *   other arguments as in pa_decode_attention.
 * bf16 only (fp32 returns PA_ERR_UNSUPPORTED); group 1, 2, 4 or 8; contexts
 * up to 2048 blocks.  A chunk longer than its context, a context beyond the
 * table, or rows outside [0, total_q) set PA_DEV_BAD_CONTEXT (its rows that
 * exist are zeros); an invalid block id sets PA_DEV_BAD_BLOCK (zeros); a
 * wait inside the kernel that runs out sets PA_DEV_WAIT_TIMEOUT.
 * Arithmetic: scores and the softmax in fp32; the softmax weights are
 * rounded to bf16 for the P.V product (their fp32 values make the row sum);
 * P.V accumulates in fp32; the output is rounded to bf16.
 */
pa_status pa_prefill_attention(void *out, const void *query, const int32_t *cu_q_lens, int total_q,
                               int max_q_len, const void *k_pool, const void *v_pool,
                               const int32_t *block_tables, int max_blocks_per_seq,
                               const int32_t *context_lens, int num_seqs, int max_context_len,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int64_t num_blocks, float scale, pa_dtype dtype,
                               int32_t *dev_status, void *stream);

/*
 * FP8 cache ("vLLM Architecture, Memory and Benchmarks Deep Dive", section 4,
 * FP8: fewer bytes per value double the effective memory bandwidth of a
 * bandwidth-bound step; "Inside vLLM: Anatomy of a High-Throughput LLM
 * Inference System", FAQ: quantized KV caches).  The pages fix no format;
 * this library's reading: every pool element is one E4M3 byte (OCP FP8:
 * sign, 4 exponent bits of bias 7, 3 mantissa bits, subnormals, no
 * infinities, 0x7f / 0xff NaN), with one scale per tensor:
 *   K = code * k_scale,  V = code * v_scale.
 * Queries, new keys and values, and outputs stay bf16.  Supported: d 128 or
 * 256, blocks of 16 or 32 tokens, Hq / Hkv in {1, 2, 4, 8}.  Pools are
 * [nb, bs, Hkv, d] bytes.
 *
 * pa_reshape_and_cache_fp8 -- the cache write: each element x of a token's
 * key (value) row is stored as the E4M3 code of x / k_scale (x / v_scale),
 * the division rounded as binary32, then rounded to the nearest code (ties
 * to the even code) with finite overflow saturating to +-448.  key, value:
 * device [num_tokens, Hkv, d] bf16; other arguments and errors as in
 * pa_reshape_and_cache; scales must be positive and finite
 * (PA_ERR_INVALID_ARG otherwise).
 */
pa_status pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_pool, void *v_pool,
                                   const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                                   int head_dim, int block_size, int64_t num_blocks,
                                   float k_scale, float v_scale, int32_t *dev_status, void *stream);

/*
 * pa_decode_attention_fp8 -- pa_decode_attention over an E4M3 cache: the
 * result is the definition of pa_decode_attention with K and V replaced by
 * their dequantised values code * k_scale and code * v_scale.  query and out
 * are bf16 [B, Hq, d]; other arguments, the workspace and the errors as in
 * pa_decode_attention (pa_decode_workspace_bytes sizes the workspace).
 * Arithmetic: both tile products run on E4M3 tensor cores with the codes as
 * stored and fp32 accumulation.  Each query row is scaled by a power of two
 * and split into two E4M3 parts, hi = e4m3(q) and lo = e4m3(q - hi): hi + lo
 * equals every query component of at least 2^-9 of its row's largest (a
 * bf16 value has 8 significant bits, hi and lo 4 each); smaller components
 * carry an absolute error of at most 2^-17 of the row's largest.  A
 * row with a non-finite component gives NaN logits.  Logits, the softmax and
 * the accumulators are fp32; the softmax weights (scaled by 2^8) are split
 * the same way for the P.V product, about 8 significant bits, and the same
 * split weights make the row sum; the output is rounded to bf16.
 */
pa_status pa_decode_attention_fp8(void *out, const void *query, const void *k_pool,
                                  const void *v_pool, const int32_t *block_tables,
                                  int max_blocks_per_seq, const int32_t *context_lens,
                                  int num_seqs, int max_context_len, int num_q_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int64_t num_blocks, float scale, float k_scale, float v_scale,
                                  void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                  void *stream);

/*
 * pa_copy_blocks -- copy whole physical blocks of both pools, the copy that
 * copy-on-write block sharing needs ("vLLM Architecture, Memory and
 * Benchmarks Deep Dive", section 2, "Copy-on-Write (CoW) Branching": rollouts
 * of one prompt share its blocks, and a block is cloned only when the
 * sequences sharing it diverge).
 *
 * For every pair i: block block_mapping[2i + 1] of k_pool and of v_pool
 * becomes a bit-exact copy of block block_mapping[2i].
 *   block_mapping  device, [num_pairs][2] int64 (source, destination).
 *                  Destinations must be distinct and must not be the source
 *                  of another pair of the same call (the copies run
 *                  concurrently).
 *   k_pool,v_pool  device, [nb, bs, Hkv, d] in `dtype` (PA_DTYPE_FP8_E4M3
 *                  for an FP8 cache).
 * A source or destination outside [0, nb) sets PA_DEV_BAD_BLOCK and that
 * pair is skipped.  num_pairs == 0 launches nothing.
 */
pa_status pa_copy_blocks(void *k_pool, void *v_pool, const int64_t *block_mapping, int num_pairs,
                         int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                         pa_dtype dtype, int32_t *dev_status, void *stream);

/*
 * pa_swap_blocks -- copy whole blocks from one pair of pools to another, for
 * paging blocks out to host memory and back ("Inside vLLM: Anatomy of a
 * High-Throughput LLM Inference System", section "Memory-Efficient KV Cache
 * Storage": blocks move between GPU and CPU memory, the less used ones paged
 * out to the host when the cache outgrows the GPU).
 *
 * For every pair i: block block_mapping[2i + 1] of dst_k_pool / dst_v_pool
 * becomes a bit-exact copy of block block_mapping[2i] of src_k_pool /
 * src_v_pool.  Either pair of pools may be device memory or pinned host
 * memory mapped into the device's address space (e.g. cudaHostAlloc on a
 * unified-addressing system); the copy runs on the GPU, asynchronously on
 * `stream`.
 *   block_mapping  device (or mapped host), [num_pairs][2] int64.
 *                  Destinations must be distinct.
 *   pools          [nb, bs, Hkv, d] in `dtype` (PA_DTYPE_FP8_E4M3 for an FP8
 *                  cache), nb given per side.
 * A block id outside its pool sets PA_DEV_BAD_BLOCK and that pair is
 * skipped.  The source and destination ranges must not overlap.  A pointer
 * the GPU cannot address as it is (pageable host memory, for instance)
 * returns PA_ERR_INVALID_ARG without a launch.
 */
pa_status pa_swap_blocks(void *dst_k_pool, void *dst_v_pool, int64_t dst_num_blocks,
                         const void *src_k_pool, const void *src_v_pool, int64_t src_num_blocks,
                         const int64_t *block_mapping, int num_pairs, int block_size,
                         int num_kv_heads, int head_dim, pa_dtype dtype, int32_t *dev_status,
                         void *stream);

/*
 * pa_decode_attention_static -- pa_decode_attention for callers that cannot
 * allocate device memory.  The pages have no counterpart to this call; it is
 * an addition of this library.
 *
 * Some callers can only hand a library their inputs and outputs: plug-in
 * interfaces of inference engines that pass no workspace, callers whose
 * device memory is owned by another framework, and code paths where an
 * allocation (which may synchronise the device) is not allowed.  This call
 * computes the same result as pa_decode_attention with a sufficient
 * workspace (bit for bit: the same kernel, grid and merge order), using
 * instead a fixed scratch array of PA_STATIC_SCRATCH_BYTES in device memory.
 * The call itself never calls cudaMalloc, cudaFree or any allocating
 * routine.
 *
 *   Arguments are those of pa_decode_attention without the workspace.
 *   Returns PA_ERR_WORKSPACE, launching nothing, when these sizes need more
 *   scratch than PA_STATIC_SCRATCH_BYTES: about 33 KB per SM for
 *   Hkv = 4, Hq / Hkv = 4, d = 256 (fits), 66 KB per SM for Hq / Hkv = 8,
 *   d = 256 (refused on a 148-SM GPU).  It refuses rather than falling back
 *   to pa_decode_attention's workspace-free decomposition, which can be much
 *   slower for long contexts: such a caller should pass a workspace.
 *   The array lives in the library's device code.  Once that code is loaded
 *   on a device, the device holds the array until the process exits.  The
 *   CUDA runtime may load it lazily (the default since CUDA 12.2): then the
 *   first call of this library on a device loads it, which places the
 *   8 MiB array in device memory (an allocation made by the driver, not by
 *   this call) and may synchronise the device.  The first call of this
 *   entry point on a device also looks up the array's device address (a
 *   CUDA runtime query).  So make a first call on each device at start-up,
 *   outside any stream capture and any section that must not allocate.
 *   All calls share the one array: calls whose kernels overlap on the GPU
 *   (other streams, other threads) race and corrupt each other's results,
 *   so serialise them.  The array keeps the last call's contents and no
 *   word of it needs to start at zero: a call counts the partial results of
 *   a split sequence in counter words tagged with that call's own tag (a
 *   word with another tag counts as zero), and reads partial results only
 *   once its own count is complete.
 */
#define PA_STATIC_SCRATCH_BYTES (8u << 20)
pa_status pa_decode_attention_static(void *out, const void *query, const void *k_pool,
                                     const void *v_pool, const int32_t *block_tables,
                                     int max_blocks_per_seq, const int32_t *context_lens,
                                     int num_seqs, int max_context_len, int num_q_heads,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int64_t num_blocks, float scale, pa_dtype dtype,
                                     int32_t *dev_status, void *stream);

/* Static description of a status code. */
const char *pa_status_string(pa_status status);

/* Number of kernels this library has launched in this process. */
unsigned long long pa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
