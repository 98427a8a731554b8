/*
 * pa_oracle.c -- plain, slow, fp64 CPU oracle for paged KV-cache decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the reference that the CUDA path is
 * checked against.  It shares no code, header, table or helper with the CUDA
 * library (paged_kv_cache_455_b200/csrc); neither side includes or links the
 * other.  Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * may load it.
 *
 * What it computes, and where the pages define it:
 *
 *   KV-size formula  M_KV = 2 * L * H_KV * d_head * T * b
 *     "Optimizing LLM Inference: A Deep Dive into vLLM's PagedAttention and
 *      Continuous Batching", section "Understanding the KV Cache Bottleneck".
 *
 *   Cache write: the new token's K and V vectors are stored in the slot of the
 *   block that was handed out for it ("vLLM Architecture, Memory and Benchmarks
 *   Deep Dive", section 2, "On-Demand Allocation"; section 1 for what the KV
 *   cache holds).  slot = physical_block * block_size + offset.
 *
 *   Gather: a per-sequence block table maps logical block j to a physical
 *   block; token t lives at (table[t / bs], t % bs).  The paged cache must look
 *   contiguous to attention ("Optimizing LLM Inference ...", section
 *   "PagedAttention: Borrowing a 50-Year-Old OS Masterpiece").
 *
 *   Attention: exact single-query softmax attention in fp64 for each query
 *   head; query head hq reads KV head hq / (Hq / Hkv) (grouped-query attention,
 *   "vLLM Architecture, Memory and Benchmarks Deep Dive", section 1: 16 layers,
 *   4 KV heads, head dim 256).  The pages do not say how query heads map onto
 *   KV heads; the reading taken here is that consecutive query heads share one
 *   KV head.
 *
 *   Partition statistics: for the context split into partitions of
 *   `partition_size` tokens, each partition's (max logit, sum of exp, normalised
 *   partial output).  Merging them with the log-sum-exp rule gives back the
 *   unsplit result; this is the flash-decoding split that the split-K kernels
 *   implement.  Written out here from its definition, per partition.
 *
 * Element types: 0 = IEEE binary32, 1 = bfloat16 (the upper 16 bits of a
 * binary32).  Both convert exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

static double elem_to_double(const void *base, int64_t index, int dtype)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[index];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[index]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Bytes of KV cache for one sequence: 2 (K and V) * layers * KV heads *
 * head dim * tokens * bytes per element. */
int64_t oracle_kv_bytes(int64_t layers, int64_t kv_heads, int64_t head_dim,
                        int64_t tokens, int64_t bytes_per_elem)
{
    return 2 * layers * kv_heads * head_dim * tokens * bytes_per_elem;
}

/* Cache write.  For every token whose slot is >= 0, copy its K and V rows
 * (all KV heads) into the pools at slot.  Pools are [nb, bs, Hkv, d].
 * Returns the number of tokens whose slot lies outside the pool (those are
 * not written); negative slots are padding and are skipped silently. */
int64_t oracle_reshape_and_cache(const void *key, const void *value,
                                 void *k_pool, void *v_pool,
                                 const int64_t *slot_mapping, int64_t num_tokens,
                                 int num_kv_heads, int head_dim, int block_size,
                                 int64_t num_blocks, int elem_size)
{
    int64_t bad = 0;
    int64_t row_bytes = (int64_t)num_kv_heads * head_dim * elem_size;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= num_blocks * block_size) {
            ++bad;
            continue;
        }
        int64_t blk = slot / block_size;
        int64_t off = slot % block_size;
        int64_t dst = (blk * block_size + off) * row_bytes;
        memcpy((char *)k_pool + dst, (const char *)key + t * row_bytes, (size_t)row_bytes);
        memcpy((char *)v_pool + dst, (const char *)value + t * row_bytes, (size_t)row_bytes);
    }
    return bad;
}

/* Checks every block id a sequence will read and its length against the
 * table width.  Returns 0 if all are valid. */
static int check_tables(const int32_t *block_tables, int max_blocks,
                        const int32_t *context_lens, int num_seqs,
                        int block_size, int64_t num_blocks)
{
    for (int b = 0; b < num_seqs; ++b) {
        int64_t ctx = context_lens[b];
        if (ctx < 0 || ctx > (int64_t)max_blocks * block_size)
            return -2;
        int64_t nblk = (ctx + block_size - 1) / block_size;
        for (int64_t j = 0; j < nblk; ++j) {
            int64_t phys = block_tables[(int64_t)b * max_blocks + j];
            if (phys < 0 || phys >= num_blocks)
                return -3;
        }
    }
    return 0;
}

/* Gathers sequence b's K and V into contiguous [ctx, Hkv, d] fp64 arrays. */
static void gather_sequence(double *kc, double *vc, const void *k_pool, const void *v_pool,
                            const int32_t *table_row, int64_t ctx, int kv_heads,
                            int head_dim, int block_size, int dtype)
{
    int64_t row = (int64_t)kv_heads * head_dim;
    for (int64_t t = 0; t < ctx; ++t) {
        int64_t phys = table_row[t / block_size];
        int64_t off = t % block_size;
        int64_t src = (phys * block_size + off) * row;
        for (int64_t e = 0; e < row; ++e) {
            kc[t * row + e] = elem_to_double(k_pool, src + e, dtype);
            vc[t * row + e] = elem_to_double(v_pool, src + e, dtype);
        }
    }
}

/* Exact attention of one query head over tokens [t_begin, t_end) of a gathered
 * sequence.  Writes m = max logit, l = sum exp(s - m) and o = sum p v / l.
 * An empty range gives m = -inf, l = 0, o = 0. */
static void attend_range(double *o, double *m_out, double *l_out, const double *q,
                         const double *kc, const double *vc, int64_t t_begin, int64_t t_end,
                         int h, int kv_heads, int head_dim, double scale)
{
    int64_t row = (int64_t)kv_heads * head_dim;
    for (int i = 0; i < head_dim; ++i)
        o[i] = 0.0;
    if (t_end <= t_begin) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return;
    }
    int64_t n = t_end - t_begin;
    double *s = (double *)malloc((size_t)n * sizeof(double));
    double m = -INFINITY;
    for (int64_t t = t_begin; t < t_end; ++t) {
        const double *k = kc + t * row + (int64_t)h * head_dim;
        double dot = 0.0;
        for (int i = 0; i < head_dim; ++i)
            dot += q[i] * k[i];
        s[t - t_begin] = scale * dot;
        if (s[t - t_begin] > m)
            m = s[t - t_begin];
    }
    double l = 0.0;
    for (int64_t t = t_begin; t < t_end; ++t) {
        double p = exp(s[t - t_begin] - m);
        const double *v = vc + t * row + (int64_t)h * head_dim;
        l += p;
        for (int i = 0; i < head_dim; ++i)
            o[i] += p * v[i];
    }
    for (int i = 0; i < head_dim; ++i)
        o[i] /= l;
    *m_out = m;
    *l_out = l;
    free(s);
}

static int set_threads(int num_threads)
{
#ifdef _OPENMP
    if (num_threads <= 0)
        num_threads = omp_get_max_threads();
    return num_threads;
#else
    (void)num_threads;
    return 1;
#endif
}

/* Threads an OpenMP region of this library would use for a request of
 * num_threads (<= 0 means all the runtime allows). */
int oracle_threads(int num_threads)
{
    return set_threads(num_threads);
}

/* Paged decode attention.  out is [B, Hq, d] fp64.  q is [B, Hq, d]; pools
 * are [nb, bs, Hkv, d]; block_tables is [B, max_blocks]; context_lens is [B].
 * A sequence of length 0 gets a zero output.  Returns 0, or a negative code
 * for invalid shapes (-1), a length above the table width (-2) or a block id
 * outside the pool (-3); nothing is written then. */
int oracle_paged_attention(double *out, const void *query, const void *k_pool,
                           const void *v_pool, const int32_t *block_tables, int max_blocks,
                           const int32_t *context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                           double scale, int dtype, int num_threads)
{
    if (num_seqs < 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
        head_dim <= 0 || block_size <= 0)
        return -1;
    int rc = check_tables(block_tables, max_blocks, context_lens, num_seqs, block_size,
                          num_blocks);
    if (rc != 0)
        return rc;
    int group = num_q_heads / num_kv_heads;
    int nt = set_threads(num_threads);
    (void)nt;

#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int b = 0; b < num_seqs; ++b) {
        int64_t ctx = context_lens[b];
        int64_t row = (int64_t)num_kv_heads * head_dim;
        double *kc = (double *)malloc((size_t)(ctx > 0 ? ctx : 1) * row * sizeof(double));
        double *vc = (double *)malloc((size_t)(ctx > 0 ? ctx : 1) * row * sizeof(double));
        double *q = (double *)malloc((size_t)head_dim * sizeof(double));
        gather_sequence(kc, vc, k_pool, v_pool, block_tables + (int64_t)b * max_blocks, ctx,
                        num_kv_heads, head_dim, block_size, dtype);
        for (int hq = 0; hq < num_q_heads; ++hq) {
            int h = hq / group;
            int64_t qoff = ((int64_t)b * num_q_heads + hq) * head_dim;
            for (int i = 0; i < head_dim; ++i)
                q[i] = elem_to_double(query, qoff + i, dtype);
            double m, l;
            attend_range(out + qoff, &m, &l, q, kc, vc, 0, ctx, h, num_kv_heads, head_dim,
                         scale);
        }
        free(q);
        free(vc);
        free(kc);
    }
    return 0;
}

/* Per-partition statistics of the same attention.  Partition p of sequence b
 * covers tokens [p*P, min((p+1)*P, ctx)).  Outputs (all fp64):
 *   part_out  [B, Hq, max_parts, d]  normalised partial output of partition p
 *   part_max  [B, Hq, max_parts]     max logit (scale * q.k) over the partition
 *   part_sum  [B, Hq, max_parts]     sum over the partition of exp(s - max)
 * Partitions at or past ceil(ctx / P) hold max = -inf, sum = 0, out = 0.
 * Same return codes as oracle_paged_attention. */
int oracle_partition_attention(double *part_out, double *part_max, double *part_sum,
                               const void *query, const void *k_pool, const void *v_pool,
                               const int32_t *block_tables, int max_blocks,
                               const int32_t *context_lens, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size,
                               int64_t num_blocks, double scale, int dtype,
                               int partition_size, int max_parts, int num_threads)
{
    if (num_seqs < 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
        head_dim <= 0 || block_size <= 0 || partition_size <= 0 || max_parts <= 0)
        return -1;
    int rc = check_tables(block_tables, max_blocks, context_lens, num_seqs, block_size,
                          num_blocks);
    if (rc != 0)
        return rc;
    for (int b = 0; b < num_seqs; ++b)
        if (((int64_t)context_lens[b] + partition_size - 1) / partition_size > max_parts)
            return -1;
    int group = num_q_heads / num_kv_heads;
    int nt = set_threads(num_threads);
    (void)nt;

#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int b = 0; b < num_seqs; ++b) {
        int64_t ctx = context_lens[b];
        int64_t row = (int64_t)num_kv_heads * head_dim;
        double *kc = (double *)malloc((size_t)(ctx > 0 ? ctx : 1) * row * sizeof(double));
        double *vc = (double *)malloc((size_t)(ctx > 0 ? ctx : 1) * row * sizeof(double));
        double *q = (double *)malloc((size_t)head_dim * sizeof(double));
        gather_sequence(kc, vc, k_pool, v_pool, block_tables + (int64_t)b * max_blocks, ctx,
                        num_kv_heads, head_dim, block_size, dtype);
        for (int hq = 0; hq < num_q_heads; ++hq) {
            int h = hq / group;
            int64_t bh = (int64_t)b * num_q_heads + hq;
            for (int i = 0; i < head_dim; ++i)
                q[i] = elem_to_double(query, bh * head_dim + i, dtype);
            for (int p = 0; p < max_parts; ++p) {
                int64_t t0 = (int64_t)p * partition_size;
                int64_t t1 = t0 + partition_size < ctx ? t0 + partition_size : ctx;
                int64_t slot = bh * max_parts + p;
                attend_range(part_out + slot * head_dim, part_max + slot, part_sum + slot, q,
                             kc, vc, t0, t1, h, num_kv_heads, head_dim, scale);
            }
        }
        free(q);
        free(vc);
        free(kc);
    }
    return 0;
}
