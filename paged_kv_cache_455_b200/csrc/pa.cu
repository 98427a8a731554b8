// pa.cu -- C ABI of the paged KV-cache decode library: argument checks,
// launch geometry and kernel dispatch.  Kernels live in pa_kernels.cuh.
//
// Split choice of pa_decode_attention: partitions of kPrefPartition tokens
// when a sequence can be longer than that and the caller's workspace holds
// the partials; with a smaller workspace the partitions grow until the
// partials fit, down to one partition per sequence (no split).
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pa.h"
#include "pa_kernels.cuh"

namespace {

using pa::DecodeParams;

std::atomic<unsigned long long> g_launches{0};

constexpr int kPrefPartition = 256;   // tokens per split-K partition (multiple of 16)

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ilog2_exact(int v)
{
    int s = 0;
    while ((1 << s) < v)
        ++s;
    return (1 << s) == v ? s : -1;
}

int round_up(int v, int m) { return ((v + m - 1) / m) * m; }

// ---------------------------------------------------------------------------
// Per-device launch facts, computed once per (device, kernel).
// ---------------------------------------------------------------------------
struct KernelSlot {
    const void *fn;
    int device;
    int grid;   // persistent grid: SMs * resident CTAs
};

std::mutex g_mu;
KernelSlot g_slots[256];
int g_nslots = 0;

pa_status persistent_grid(const void *fn, int smem_bytes, int *grid_out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PA_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        for (int i = 0; i < g_nslots; ++i)
            if (g_slots[i].fn == fn && g_slots[i].device == dev) {
                *grid_out = g_slots[i].grid;
                return PA_OK;
            }
    }
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
        cudaSuccess)
        return PA_ERR_CUDA;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return PA_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, pa::kThreads, smem_bytes) !=
        cudaSuccess)
        return PA_ERR_CUDA;
    if (per_sm < 1)
        return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_nslots < 256)
        g_slots[g_nslots++] = KernelSlot{fn, dev, sms * per_sm};
    *grid_out = sms * per_sm;
    return PA_OK;
}

// ---------------------------------------------------------------------------
// Decode dispatch over (dtype, head_dim, group, math)
// ---------------------------------------------------------------------------
template <typename T, int D, int G, bool MMA>
pa_status launch_decode_t(const DecodeParams &p, int64_t items_upper, cudaStream_t stream)
{
    const void *fn = reinterpret_cast<const void *>(&pa::decode_kernel<T, D, G, MMA>);
    constexpr int smem = pa::Layout<T, D, G>::kSmem;
    int grid = 0;
    pa_status st = persistent_grid(fn, smem, &grid);
    if (st != PA_OK)
        return st;
    if (items_upper < grid)
        grid = (int)(items_upper > 0 ? items_upper : 1);
    pa::decode_kernel<T, D, G, MMA><<<grid, pa::kThreads, smem, stream>>>(p);
    ++g_launches;
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int D, bool MMA>
pa_status launch_decode_g(const DecodeParams &p, int group, int64_t items, cudaStream_t s)
{
    switch (group) {
    case 1: return launch_decode_t<T, D, 1, MMA>(p, items, s);
    case 2: return launch_decode_t<T, D, 2, MMA>(p, items, s);
    case 4: return launch_decode_t<T, D, 4, MMA>(p, items, s);
    case 8: return launch_decode_t<T, D, 8, MMA>(p, items, s);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T, bool MMA>
pa_status launch_decode_d(const DecodeParams &p, int head_dim, int group, int64_t items,
                          cudaStream_t s)
{
    switch (head_dim) {
    case 64: return launch_decode_g<T, 64, MMA>(p, group, items, s);
    case 128: return launch_decode_g<T, 128, MMA>(p, group, items, s);
    case 256: return launch_decode_g<T, 256, MMA>(p, group, items, s);
    default: return PA_ERR_UNSUPPORTED;
    }
}

// bf16 uses the tensor-core tile math unless PA_DECODE_MATH=simt is set
// (kept to compare the two on the same data).
bool bf16_use_mma()
{
    const char *v = std::getenv("PA_DECODE_MATH");
    return !(v && std::strcmp(v, "simt") == 0);
}

pa_status launch_decode(const DecodeParams &p, pa_dtype dtype, int head_dim, int group,
                        int64_t items, cudaStream_t s)
{
    if (dtype == PA_DTYPE_F32)
        return launch_decode_d<float, false>(p, head_dim, group, items, s);
    if (bf16_use_mma())
        return launch_decode_d<__nv_bfloat16, true>(p, head_dim, group, items, s);
    return launch_decode_d<__nv_bfloat16, false>(p, head_dim, group, items, s);
}

// ---------------------------------------------------------------------------
// Shared argument checks of the attention calls
// ---------------------------------------------------------------------------
pa_status check_attention_args(const void *out, const void *query, const void *k_pool,
                               const void *v_pool, const int32_t *block_tables,
                               int max_blocks, const int32_t *context_lens, int num_seqs,
                               int max_context_len, int num_q_heads, int num_kv_heads,
                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                               int *group_out, int *bs_log2_out)
{
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks <= 0 || max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16)
        return PA_ERR_UNSUPPORTED;
    const int group = num_q_heads / num_kv_heads;
    if (group != 1 && group != 2 && group != 4 && group != 8)
        return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return PA_ERR_UNSUPPORTED;
    const int bs_log2 = ilog2_exact(block_size);
    if (block_size < 4 || block_size > 32 || bs_log2 < 0)
        return PA_ERR_UNSUPPORTED;
    if ((int64_t)max_context_len > (int64_t)max_blocks * block_size)
        return PA_ERR_INVALID_ARG;
    if (num_blocks > (int64_t)INT32_MAX)
        return PA_ERR_INVALID_ARG;   // block ids are int32
    if (num_seqs > 0) {
        if (!out || !query || !k_pool || !v_pool || !block_tables || !context_lens)
            return PA_ERR_INVALID_ARG;
        if (!aligned16(out) || !aligned16(query) || !aligned16(k_pool) || !aligned16(v_pool))
            return PA_ERR_INVALID_ARG;
    }
    *group_out = group;
    *bs_log2_out = bs_log2;
    return PA_OK;
}

DecodeParams make_params(void *out, const void *query, const void *k_pool, const void *v_pool,
                         const int32_t *block_tables, int max_blocks,
                         const int32_t *context_lens, int num_seqs, int num_q_heads,
                         int num_kv_heads, int block_size, int bs_log2, int64_t num_blocks,
                         float scale, int partition_size, int max_parts, float *tmp_out,
                         float *max_logits, float *exp_sums, int always_partials,
                         int32_t *dev_status)
{
    DecodeParams p;
    p.out = out;
    p.q = query;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.tmp_out = tmp_out;
    p.max_logits = max_logits;
    p.exp_sums = exp_sums;
    p.dev_status = dev_status;
    p.num_blocks = num_blocks;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.max_blocks = max_blocks;
    p.block_size = block_size;
    p.bs_log2 = bs_log2;
    p.partition_size = partition_size;
    p.max_parts = max_parts;
    const int64_t cap = std::min<int64_t>((int64_t)max_blocks * block_size,
                                          (int64_t)max_parts * partition_size);
    p.ctx_cap = (int)std::min<int64_t>(cap, INT32_MAX);
    p.always_partials = always_partials;
    p.scale_log2 = scale * pa::kLog2e;
    return p;
}

template <typename T>
pa_status launch_reduce_t(const pa::ReduceParams &rp, int head_dim, int num_seqs,
                          cudaStream_t stream)
{
    const int64_t grid = (int64_t)num_seqs * rp.num_q_heads;
    if (grid > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    pa::reduce_kernel<T><<<(unsigned)grid, 128, 0, stream>>>(rp, head_dim);
    ++g_launches;
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status launch_reduce(void *out, const float *tmp_out, const float *max_logits,
                        const float *exp_sums, const int32_t *context_lens, int num_seqs,
                        int num_q_heads, int head_dim, int partition_size, int max_parts,
                        int ctx_cap, pa_dtype dtype, cudaStream_t stream)
{
    pa::ReduceParams rp;
    rp.out = out;
    rp.tmp_out = tmp_out;
    rp.max_logits = max_logits;
    rp.exp_sums = exp_sums;
    rp.context_lens = context_lens;
    rp.num_seqs = num_seqs;
    rp.num_q_heads = num_q_heads;
    rp.partition_size = partition_size;
    rp.max_parts = max_parts;
    rp.ctx_cap = ctx_cap;
    if (dtype == PA_DTYPE_F32)
        return launch_reduce_t<float>(rp, head_dim, num_seqs, stream);
    return launch_reduce_t<__nv_bfloat16>(rp, head_dim, num_seqs, stream);
}

size_t splitk_bytes(int64_t num_seqs, int64_t num_q_heads, int64_t head_dim, int64_t parts)
{
    return (size_t)(num_seqs * num_q_heads * parts * (head_dim + 2) * 4);
}

}  // namespace

extern "C" {

const char *pa_status_string(pa_status status)
{
    switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported head_dim, block_size, group or dtype";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
    }
}

unsigned long long pa_launch_count(void) { return g_launches.load(); }

int pa_num_partitions(int max_context_len, int partition_size)
{
    if (partition_size <= 0 || max_context_len <= 0)
        return 1;
    return (int)(((int64_t)max_context_len + partition_size - 1) / partition_size);
}

size_t pa_splitk_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_partitions)
{
    if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_partitions <= 0)
        return 0;
    return splitk_bytes(num_seqs, num_q_heads, head_dim, max_partitions);
}

size_t pa_decode_workspace_bytes(int num_seqs, int num_q_heads, int head_dim,
                                 int max_context_len)
{
    if (max_context_len <= kPrefPartition)
        return 0;
    return pa_splitk_workspace_bytes(num_seqs, num_q_heads, head_dim,
                                     pa_num_partitions(max_context_len, kPrefPartition));
}

pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_pool, void *v_pool,
                               const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                               int32_t *dev_status, void *stream)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16)
        return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return PA_ERR_UNSUPPORTED;
    if (ilog2_exact(block_size) < 0 || block_size < 4 || block_size > 32)
        return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0)
        return PA_OK;
    if (!key || !value || !k_pool || !v_pool || !slot_mapping)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_pool) || !aligned16(v_pool))
        return PA_ERR_INVALID_ARG;
    pa::CacheParams p;
    p.key = key;
    p.value = value;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.slot_mapping = slot_mapping;
    p.dev_status = dev_status;
    p.num_slots = num_blocks * block_size;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.row_bytes = head_dim * (dtype == PA_DTYPE_F32 ? 4 : 2);
    const int64_t rows = (int64_t)num_tokens * num_kv_heads * 2;
    const int64_t blocks = (rows + 7) / 8;   // 8 warps per CTA
    if (blocks > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    pa::cache_write_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    ++g_launches;
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_decode_splitk(void *out, const void *query, const void *k_pool, const void *v_pool,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int num_seqs, int max_context_len,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int64_t num_blocks, float scale, pa_dtype dtype, int partition_size,
                           int max_partitions, float *tmp_out, float *max_logits,
                           float *exp_sums, int32_t *dev_status, void *stream)
{
    int group = 0, bs_log2 = 0;
    pa_status st = check_attention_args(out, query, k_pool, v_pool, block_tables,
                                        max_blocks_per_seq, context_lens, num_seqs,
                                        max_context_len, num_q_heads, num_kv_heads, head_dim,
                                        block_size, num_blocks, dtype, &group, &bs_log2);
    if (st != PA_OK)
        return st;
    if (partition_size <= 0 || partition_size % pa::kTile != 0 || max_partitions <= 0)
        return PA_ERR_INVALID_ARG;
    if (max_partitions < pa_num_partitions(max_context_len, partition_size))
        return PA_ERR_WORKSPACE;
    if (num_seqs == 0)
        return PA_OK;
    if (!tmp_out || !max_logits || !exp_sums)
        return PA_ERR_INVALID_ARG;
    const int64_t items = (int64_t)num_seqs * num_kv_heads * max_partitions;
    if (items > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    DecodeParams p = make_params(out, query, k_pool, v_pool, block_tables, max_blocks_per_seq,
                                 context_lens, num_seqs, num_q_heads, num_kv_heads, block_size,
                                 bs_log2, num_blocks, scale, partition_size, max_partitions,
                                 tmp_out, max_logits, exp_sums, 1, dev_status);
    return launch_decode(p, dtype, head_dim, group, items, static_cast<cudaStream_t>(stream));
}

pa_status pa_splitk_reduce(void *out, const float *tmp_out, const float *max_logits,
                           const float *exp_sums, const int32_t *context_lens, int num_seqs,
                           int num_q_heads, int head_dim, int partition_size,
                           int max_partitions, pa_dtype dtype, void *stream)
{
    if (num_seqs < 0 || num_q_heads <= 0 || partition_size <= 0 ||
        partition_size % pa::kTile != 0 || max_partitions <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16)
        return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0)
        return PA_OK;
    if (!out || !tmp_out || !max_logits || !exp_sums || !context_lens)
        return PA_ERR_INVALID_ARG;
    const int64_t cap = (int64_t)max_partitions * partition_size;
    return launch_reduce(out, tmp_out, max_logits, exp_sums, context_lens, num_seqs, num_q_heads,
                         head_dim, partition_size, max_partitions,
                         (int)std::min<int64_t>(cap, INT32_MAX), dtype,
                         static_cast<cudaStream_t>(stream));
}

pa_status pa_decode_attention(void *out, const void *query, const void *k_pool,
                              const void *v_pool, const int32_t *block_tables,
                              int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                              int max_context_len, int num_q_heads, int num_kv_heads,
                              int head_dim, int block_size, int64_t num_blocks, float scale,
                              pa_dtype dtype, void *workspace, size_t workspace_bytes,
                              int32_t *dev_status, void *stream)
{
    int group = 0, bs_log2 = 0;
    pa_status st = check_attention_args(out, query, k_pool, v_pool, block_tables,
                                        max_blocks_per_seq, context_lens, num_seqs,
                                        max_context_len, num_q_heads, num_kv_heads, head_dim,
                                        block_size, num_blocks, dtype, &group, &bs_log2);
    if (st != PA_OK)
        return st;
    if (num_seqs == 0)
        return PA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // Partition size: kPrefPartition if the partials fit the workspace, else
    // the smallest multiple of 16 whose partials fit, else no split.
    const int full = round_up(max_context_len > 0 ? max_context_len : 1, pa::kTile);
    int P = full;
    int parts = 1;
    if (max_context_len > kPrefPartition && workspace != nullptr) {
        const size_t per_part = splitk_bytes(num_seqs, num_q_heads, head_dim, 1);
        const int64_t fit = (int64_t)(workspace_bytes / per_part);
        const int want = pa_num_partitions(max_context_len, kPrefPartition);
        const int64_t use = std::min<int64_t>(fit, want);
        if (use >= 2) {
            P = round_up(pa_num_partitions(max_context_len, (int)use), pa::kTile);
            P = std::max(P, kPrefPartition);
            parts = pa_num_partitions(max_context_len, P);
        }
    }
    const int64_t items = (int64_t)num_seqs * num_kv_heads * parts;
    if (items > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    float *tmp = nullptr, *ml = nullptr, *es = nullptr;
    if (parts > 1) {
        if (!aligned16(workspace))
            return PA_ERR_INVALID_ARG;
        tmp = static_cast<float *>(workspace);
        ml = tmp + (int64_t)num_seqs * num_q_heads * parts * head_dim;
        es = ml + (int64_t)num_seqs * num_q_heads * parts;
    }
    DecodeParams p = make_params(out, query, k_pool, v_pool, block_tables, max_blocks_per_seq,
                                 context_lens, num_seqs, num_q_heads, num_kv_heads, block_size,
                                 bs_log2, num_blocks, scale, P, parts, tmp, ml, es, 0, dev_status);
    st = launch_decode(p, dtype, head_dim, group, items, s);
    if (st != PA_OK || parts == 1)
        return st;
    return launch_reduce(out, tmp, ml, es, context_lens, num_seqs, num_q_heads, head_dim, P,
                         parts, p.ctx_cap, dtype, s);
}

}  // extern "C"
