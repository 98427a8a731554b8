// pa_kernels.cuh -- sm_100a kernels of the paged KV-cache decode library.
//
// Kernels
//   cache_write_kernel   new token's K/V rows -> their pool slots (bit copy).
//   decode_kernel        persistent split-K paged attention: every (sequence,
//                        KV head, context partition) is one work item; each
//                        CTA walks items with a grid stride.  Per warp, K/V
//                        tiles of 16 tokens stream into shared memory through
//                        bulk copies (one per 16-token row slice, addressed
//                        through the block table) completed on mbarriers,
//                        SPW tiles in flight.  All query heads of the GQA
//                        group are served from one read of each K/V tile.
//   reduce_kernel        log-sum-exp merge of the partitions of a sequence.
//
// The math of a tile is one of two policies:
//   SimtMath  fp32 FMAs, one token row spread over a warp (or part of one),
//             warp-shuffle dot products; used for fp32 data (and, on request,
//             for bf16).
//   MmaMath   bf16 tensor-core MMAs (m16n8k16, fp32 accumulate): S = K Q^T
//             with the group's heads as the N = 8 columns, then
//             O^T += V^T P^T with P transposed in registers by movmatrix.
// Both keep an online softmax in fp32 in the log2 domain.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <type_traits>

#include "pa.h"
#include "pa_ptx.cuh"

namespace pa {

constexpr int kThreads = 128;               // 4 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kTile = 16;                   // tokens per tile (= MMA M / K)
constexpr int kSmemBudget = 227 * 1024;     // opt-in dynamic shared memory per CTA
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded copy waits: 2 s
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned kFull = 0xffffffffu;

struct DecodeParams {
    void *out;
    const void *q;
    const void *k_pool;
    const void *v_pool;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *tmp_out;
    float *max_logits;
    float *exp_sums;
    int32_t *dev_status;
    int64_t num_blocks;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int max_blocks;
    int block_size;
    int bs_log2;
    int partition_size;     // multiple of kTile
    int max_parts;
    int ctx_cap;            // lengths above this are invalid
    int always_partials;    // write partials even for single-partition sequences
    float scale_log2;       // softmax scale * log2(e)
};

struct CacheParams {
    const void *key;
    const void *value;
    void *k_pool;
    void *v_pool;
    const int64_t *slot_mapping;
    int32_t *dev_status;
    int64_t num_slots;      // nb * bs
    int num_tokens;
    int num_kv_heads;
    int row_bytes;          // d * element size
};

struct ReduceParams {
    void *out;
    const float *tmp_out;
    const float *max_logits;
    const float *exp_sums;
    const int32_t *context_lens;
    int num_seqs;
    int num_q_heads;
    int partition_size;
    int max_parts;
    int ctx_cap;
};

__device__ __forceinline__ void report(int32_t *status, int bit)
{
    if (status)
        atomicOr(status, bit);
}

// =====================================================================
// Cache write: one warp per (token, KV head, K|V) row, 16-byte copies.
// =====================================================================
__global__ void __launch_bounds__(256) cache_write_kernel(const CacheParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nrows = (int64_t)p.num_tokens * p.num_kv_heads * 2;
    if (row >= nrows)
        return;
    const int kv = (int)(row & 1);
    const int64_t th = row >> 1;
    const int64_t t = th / p.num_kv_heads;
    const int64_t h = th - t * p.num_kv_heads;
    const int64_t slot = p.slot_mapping[t];
    if (slot < 0)
        return;
    if (slot >= p.num_slots) {
        if (lane == 0 && h == 0 && kv == 0)
            report(p.dev_status, PA_DEV_BAD_SLOT);
        return;
    }
    const int4 *src = reinterpret_cast<const int4 *>(
        static_cast<const uint8_t *>(kv ? p.value : p.key) + (t * p.num_kv_heads + h) * p.row_bytes);
    int4 *dst = reinterpret_cast<int4 *>(static_cast<uint8_t *>(kv ? p.v_pool : p.k_pool) +
                                         (slot * p.num_kv_heads + h) * p.row_bytes);
    const int n16 = p.row_bytes >> 4;
    for (int c = lane; c < n16; c += 32)
        dst[c] = __ldg(src + c);
}

// =====================================================================
// Work items: (sequence b, context partition, KV head h), enumerated
// sequence-major, then partition, then head.
// =====================================================================
__device__ __forceinline__ int eff_ctx(int ctx, int cap) { return (ctx < 0 || ctx > cap) ? 0 : ctx; }
__device__ __forceinline__ int num_parts(int ctx, int P) { return ctx <= 0 ? 1 : (ctx + P - 1) / P; }

struct SeqCursor {
    int b;         // current sequence
    int base;      // first item of sequence b
    int cnt;       // items of sequence b (= parts * Hkv)
    int ctx;       // effective length of b
    int ctx_raw;   // length as given
};

struct Item {
    int b, h, part, t0, t1, ctx, ctx_raw;
};

__device__ __forceinline__ void cursor_reset(SeqCursor &c)
{
    c.b = -1;
    c.base = 0;
    c.cnt = 0;
    c.ctx = 0;
    c.ctx_raw = 0;
}

// Total number of items (every lane gets it).
__device__ int count_items(const DecodeParams &p, int lane)
{
    int sum = 0;
    for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
        const int b = b0 + lane;
        if (b < p.num_seqs)
            sum += num_parts(eff_ctx(p.context_lens[b], p.ctx_cap), p.partition_size) *
                   p.num_kv_heads;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        sum += __shfl_xor_sync(kFull, sum, o);
    return sum;
}

// Moves the cursor forward to the sequence holding item g (g must not be
// below the cursor's base and must be below the total).  Warp-cooperative:
// 32 sequences per step with a shuffle prefix sum.
__device__ void cursor_seek(SeqCursor &c, int g, const DecodeParams &p, int lane)
{
    while (g >= c.base + c.cnt) {
        const int base = c.base + c.cnt;
        const int b0 = c.b + 1;
        const int bb = b0 + lane;
        const bool in = bb < p.num_seqs;
        const int raw = in ? p.context_lens[bb] : 0;
        const int ctx = eff_ctx(raw, p.ctx_cap);
        const int cnt = in ? num_parts(ctx, p.partition_size) * p.num_kv_heads : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFull, incl, o);
            if (lane >= o)
                incl += v;
        }
        const unsigned hit = __ballot_sync(kFull, in && g < base + incl);
        const int L = hit ? (__ffs(hit) - 1) : 31;
        c.b = b0 + L;
        c.base = base + __shfl_sync(kFull, incl - cnt, L);
        c.cnt = __shfl_sync(kFull, cnt, L);
        c.ctx = __shfl_sync(kFull, ctx, L);
        c.ctx_raw = __shfl_sync(kFull, raw, L);
    }
}

__device__ __forceinline__ Item locate(SeqCursor &c, int g, const DecodeParams &p, int lane)
{
    cursor_seek(c, g, p, lane);
    Item it;
    const int local = g - c.base;
    it.b = c.b;
    it.part = local / p.num_kv_heads;
    it.h = local - it.part * p.num_kv_heads;
    it.ctx = c.ctx;
    it.ctx_raw = c.ctx_raw;
    it.t0 = it.part * p.partition_size;
    it.t1 = min(it.t0 + p.partition_size, it.ctx);
    return it;
}

__device__ __forceinline__ int item_tiles(const Item &it)
{
    return it.t1 > it.t0 ? (it.t1 - it.t0 + kTile - 1) / kTile : 0;
}

// =====================================================================
// Shared-memory layout of the decode kernel
// =====================================================================
template <typename T, int D, int G>
struct Layout {
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kRowStride = kRowBytes + 16;          // pad: conflict-free ldmatrix
    static constexpr int kHalf = kTile * kRowStride;            // K (or V) part of a stage
    static constexpr int kStage = 2 * kHalf;
    static constexpr int kMergeFloats = G * D + 2 * G + 1;      // acc, m, l, bad flag
    static constexpr int kMergeBytes = kWarps * kMergeFloats * 4;
    static constexpr int kScoreBytes = kWarps * kTile * G * 4;
    static constexpr int kFixed = ((kMergeBytes + kScoreBytes + 15) / 16) * 16 + 8 * kWarps * 4;
    static constexpr int kSpwFit = (kSmemBudget - kFixed) / (kWarps * kStage);
    static constexpr int kSPW = kSpwFit > 4 ? 4 : kSpwFit;     // stages per warp
    static_assert(kSPW >= 1, "a stage must fit");
    static constexpr int kStagesBytes = kWarps * kSPW * kStage;
    static constexpr int kMergeOff = kStagesBytes;
    static constexpr int kScoreOff = kMergeOff + kMergeBytes;
    static constexpr int kBarOff = ((kScoreOff + kScoreBytes + 15) / 16) * 16;
    static constexpr int kSmem = kBarOff + 8 * kWarps * kSPW;
    static_assert(kSmem <= kSmemBudget, "shared memory over budget");
};

// =====================================================================
// Tile math, CUDA cores
// =====================================================================
template <typename T, int D, int G>
struct SimtMath {
    static constexpr int VEC = 16 / (int)sizeof(T);   // elements per 16-byte chunk
    static constexpr int NCH = D / VEC;                // chunks per row
    static constexpr int LPR = NCH < 32 ? NCH : 32;    // lanes per row
    static constexpr int RPI = 32 / LPR;               // rows side by side
    static constexpr int CPL = NCH / LPR;              // chunks per lane
    static constexpr int NE = CPL * VEC;               // elements per lane
    static constexpr int RPL = kTile / RPI;            // rows per lane per tile
    using L = Layout<T, D, G>;

    float q[G][NE];
    float acc[G][NE];
    float m[G];   // running max, log2 domain (warp-uniform)
    float l[G];   // running sum over this lane's rows

    __device__ __forceinline__ static void load_chunk(const void *src, float (&x)[VEC])
    {
        const uint4 u = *reinterpret_cast<const uint4 *>(src);
        if constexpr (sizeof(T) == 4) {
            x[0] = __uint_as_float(u.x);
            x[1] = __uint_as_float(u.y);
            x[2] = __uint_as_float(u.z);
            x[3] = __uint_as_float(u.w);
        } else {
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[2 * i] = ptx::bf16lo_to_f32(w[i]);
                x[2 * i + 1] = ptx::bf16hi_to_f32(w[i]);
            }
        }
    }

    __device__ __forceinline__ void begin(const T *qhead, float scale_log2, int lane)
    {
        const int li = lane % LPR;
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                float x[VEC];
                load_chunk(qhead + g * D + (c * LPR + li) * VEC, x);
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    q[g][c * VEC + v] = x[v] * scale_log2;
                    acc[g][c * VEC + v] = 0.f;
                }
            }
            m[g] = -INFINITY;
            l[g] = 0.f;
        }
    }

    __device__ __forceinline__ void tile(const uint8_t *ks, const uint8_t *vs, int n,
                                         float *scores, int lane)
    {
        const int li = lane % LPR;
        const int rg = lane / LPR;
        float tmax[G];
#pragma unroll
        for (int g = 0; g < G; ++g)
            tmax[g] = -INFINITY;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const int r = rg + i * RPI;
            float part[G];
#pragma unroll
            for (int g = 0; g < G; ++g)
                part[g] = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                float k[VEC];
                load_chunk(ks + r * L::kRowStride + (c * LPR + li) * 16, k);
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int v = 0; v < VEC; ++v)
                        part[g] = fmaf(q[g][c * VEC + v], k[v], part[g]);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1)
                    part[g] += __shfl_xor_sync(kFull, part[g], o);
                const float s = r < n ? part[g] : -INFINITY;
                tmax[g] = fmaxf(tmax[g], s);
                if (li == 0)
                    scores[r * G + g] = s;
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int o = LPR; o < 32; o <<= 1)
                tmax[g] = fmaxf(tmax[g], __shfl_xor_sync(kFull, tmax[g], o));
        }
        __syncwarp();
        float ref[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mn = fmaxf(m[g], tmax[g]);
            const float alpha = mn == -INFINITY ? 1.f : ptx::ex2(m[g] - mn);
            m[g] = mn;
            ref[g] = mn == -INFINITY ? 0.f : mn;
            l[g] *= alpha;
#pragma unroll
            for (int e = 0; e < NE; ++e)
                acc[g][e] *= alpha;
        }
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const int r = rg + i * RPI;
            if (r < n) {
                float pr[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    pr[g] = ptx::ex2(scores[r * G + g] - ref[g]);
                    l[g] += pr[g];
                }
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    float v[VEC];
                    load_chunk(vs + r * L::kRowStride + (c * LPR + li) * 16, v);
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int e = 0; e < VEC; ++e)
                            acc[g][c * VEC + e] = fmaf(pr[g], v[e], acc[g][c * VEC + e]);
                }
            }
        }
        __syncwarp();
    }

    // Writes this warp's (acc, m, l) into its merge row; lanes of row group 0
    // hold the sums over all row groups.
    __device__ __forceinline__ void finish(float *mrow, int lane)
    {
        const int li = lane % LPR;
        const int rg = lane / LPR;
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int o = LPR; o < 32; o <<= 1) {
                l[g] += __shfl_xor_sync(kFull, l[g], o);
#pragma unroll
                for (int e = 0; e < NE; ++e)
                    acc[g][e] += __shfl_xor_sync(kFull, acc[g][e], o);
            }
        }
        if (rg == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int c = 0; c < CPL; ++c)
#pragma unroll
                    for (int v = 0; v < VEC; ++v)
                        mrow[g * D + (c * LPR + li) * VEC + v] = acc[g][c * VEC + v];
        }
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                mrow[G * D + g] = m[g];
                mrow[G * D + G + g] = l[g];
            }
        }
    }
};

// =====================================================================
// Tile math, bf16 tensor cores (warp-level MMA)
//
// Fragment maps (r = lane / 4, c = lane % 4):
//   S = K Q^T, M = 16 tokens, N = 8 heads (G real), K = d in steps of 16.
//     S frag: s0,s1 = S[tok r][head 2c, 2c+1], s2,s3 = S[tok r+8][...].
//   O^T += V^T P^T, M = 16 d-rows per tile mt, N = 8 heads, K = 16 tokens.
//     P^T frag from movmatrix of the packed S frag; O^T frag:
//     a0,a1 = O^T[d 16mt+r][head 2c, 2c+1], a2,a3 = O^T[d 16mt+r+8][...].
// Each lane owns heads 2c and 2c+1 in both maps, so the running max, sum and
// rescale of those heads never leave the lane (apart from the max reduce).
// =====================================================================
template <int D, int G>
struct MmaMath {
    static_assert(G <= 8, "group must fit the N = 8 MMA");
    static constexpr int KS = D / 16;
    using L = Layout<__nv_bfloat16, D, G>;

    uint32_t qf[KS][2];
    float acc[KS][4];
    float m[2];
    float l[2];

    __device__ __forceinline__ void begin(const __nv_bfloat16 *qhead, float, int lane)
    {
        const int r = lane >> 2, c = lane & 3;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            if (r < G) {
                const uint32_t *qr = reinterpret_cast<const uint32_t *>(qhead + r * D + 16 * k);
                qf[k][0] = qr[c];
                qf[k][1] = qr[4 + c];
            } else {
                qf[k][0] = 0u;
                qf[k][1] = 0u;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[k][i] = 0.f;
        }
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
    }

    __device__ __forceinline__ void tile(uint32_t ks, uint32_t vs, int n, float scale_log2,
                                         int lane)
    {
        const int r = lane >> 2;
        // ---- S = K Q^T (two accumulation chains)
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t kaddr = ks + (lane & 15) * L::kRowStride + (lane >> 4) * 16;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            uint32_t a[4];
            ptx::ldsm_x4(kaddr + k * 32, a);
            if (k & 1)
                ptx::mma_bf16_16816(sb, a, qf[k][0], qf[k][1]);
            else
                ptx::mma_bf16_16816(sa, a, qf[k][0], qf[k][1]);
        }
        float s[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            s[i] = (sa[i] + sb[i]) * scale_log2;
        if (r >= n) {
            s[0] = -INFINITY;
            s[1] = -INFINITY;
        }
        if (r + 8 >= n) {
            s[2] = -INFINITY;
            s[3] = -INFINITY;
        }
        // ---- online softmax for heads 2c, 2c+1
        float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o));
        }
        const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
        const float al0 = mn0 == -INFINITY ? 1.f : ptx::ex2(m[0] - mn0);
        const float al1 = mn1 == -INFINITY ? 1.f : ptx::ex2(m[1] - mn1);
        const float rf0 = mn0 == -INFINITY ? 0.f : mn0;
        const float rf1 = mn1 == -INFINITY ? 0.f : mn1;
        m[0] = mn0;
        m[1] = mn1;
        const uint32_t p01 = ptx::pack_bf16x2(ptx::ex2(s[0] - rf0), ptx::ex2(s[1] - rf1));
        const uint32_t p23 = ptx::pack_bf16x2(ptx::ex2(s[2] - rf0), ptx::ex2(s[3] - rf1));
        // the sum uses the same rounded weights as the MMA
        l[0] = l[0] * al0 + ptx::bf16lo_to_f32(p01) + ptx::bf16lo_to_f32(p23);
        l[1] = l[1] * al1 + ptx::bf16hi_to_f32(p01) + ptx::bf16hi_to_f32(p23);
        if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                acc[k][0] *= al0;
                acc[k][1] *= al1;
                acc[k][2] *= al0;
                acc[k][3] *= al1;
            }
        }
        const uint32_t b0 = ptx::movmatrix_trans(p01);
        const uint32_t b1 = ptx::movmatrix_trans(p23);
        // ---- O^T += V^T P^T
        const uint32_t vaddr =
            vs + ((lane & 7) + ((lane >> 4) << 3)) * L::kRowStride + ((lane >> 3) & 1) * 16;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            uint32_t a[4];
            ptx::ldsm_x4_trans(vaddr + k * 32, a);
            ptx::mma_bf16_16816(acc[k], a, b0, b1);
        }
    }

    __device__ __forceinline__ void finish(float *mrow, int lane)
    {
        const int r = lane >> 2, c = lane & 3;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l[0] += __shfl_xor_sync(kFull, l[0], o);
            l[1] += __shfl_xor_sync(kFull, l[1], o);
        }
        const int h0 = 2 * c, h1 = 2 * c + 1;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int d0 = 16 * k + r;
            if (h0 < G) {
                mrow[h0 * D + d0] = acc[k][0];
                mrow[h0 * D + d0 + 8] = acc[k][2];
            }
            if (h1 < G) {
                mrow[h1 * D + d0] = acc[k][1];
                mrow[h1 * D + d0 + 8] = acc[k][3];
            }
        }
        if (r == 0) {
            if (h0 < G) {
                mrow[G * D + h0] = m[0];
                mrow[G * D + G + h0] = l[0];
            }
            if (h1 < G) {
                mrow[G * D + h1] = m[1];
                mrow[G * D + G + h1] = l[1];
            }
        }
    }
};

// =====================================================================
// Decode kernel
// =====================================================================
template <typename T>
__device__ __forceinline__ void store_out(T *dst, float v);
template <>
__device__ __forceinline__ void store_out<float>(float *dst, float v) { *dst = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16 *dst, float v)
{
    *dst = __float2bfloat16_rn(v);
}

template <typename T, int D, int G, bool MMA>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p)
{
    using L = Layout<T, D, G>;
    constexpr int SPW = L::kSPW;
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    float *merge = reinterpret_cast<float *>(smem + L::kMergeOff);
    float *scores = reinterpret_cast<float *>(smem + L::kScoreOff) + warp * kTile * G;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);

    // Rows that are never copied (past a sequence's end) must hold finite
    // values: their weight is exactly 0 and 0 * finite = 0 in the MMA.
    for (int i = threadIdx.x; i < L::kStagesBytes / 16; i += kThreads)
        reinterpret_cast<int4 *>(smem)[i] = make_int4(0, 0, 0, 0);
    if (threadIdx.x < kWarps * SPW)
        ptx::mbar_init(ptx::smem_u32(&bars[threadIdx.x]), 1);
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    __syncthreads();

    const int total = count_items(p, lane);
    const uint32_t stage0 = ptx::smem_u32(smem + warp * SPW * L::kStage);
    const uint32_t bar0 = ptx::smem_u32(&bars[warp * SPW]);
    const uint8_t *kpool = static_cast<const uint8_t *>(p.k_pool);
    const uint8_t *vpool = static_cast<const uint8_t *>(p.v_pool);
    const int Hkv = p.num_kv_heads;
    const uint64_t policy = ptx::policy_evict_first();

    // ---------------- producer: this warp's job stream, SPW jobs ahead
    SeqCursor pc;
    cursor_reset(pc);
    int pk = -1, pj = 0, pnt = 0;
    bool pdone = false;
    Item pit{};
    uint32_t badmask = 0;   // stage s holds a tile with a bad block id
    uint32_t issued = 0, consumed = 0;
    bool aborted = false;

    auto next_job = [&](Item &it, int &j) -> bool {
        while (!pdone) {
            if (pk >= 0 && pj < pnt) {
                it = pit;
                j = pj;
                pj += kWarps;
                return true;
            }
            ++pk;
            const long long g = (long long)blockIdx.x + (long long)pk * gridDim.x;
            if (g >= total) {
                pdone = true;
                break;
            }
            pit = locate(pc, (int)g, p, lane);
            pnt = item_tiles(pit);
            pj = warp;
        }
        return false;
    };

    auto issue = [&](const Item &it, int j, int s) {
        const int tb = it.t0 + j * kTile;
        const int n = min(kTile, it.t1 - tb);
        const int row = lane & 15;
        const int isv = lane >> 4;
        const int t = tb + row;
        const bool valid = row < n;
        int phys = 0;
        if (valid)
            phys = p.block_tables[(int64_t)it.b * p.max_blocks + (t >> p.bs_log2)];
        const bool bad = valid && (phys < 0 || (int64_t)phys >= p.num_blocks);
        const bool go = valid && !bad;
        const unsigned gom = __ballot_sync(kFull, go);
        if (__ballot_sync(kFull, bad))
            badmask |= 1u << s;
        const uint32_t bar = bar0 + 8u * s;
        if (lane == 0)
            ptx::mbar_arrive_expect_tx(bar, (uint32_t)__popc(gom) * L::kRowBytes);
        __syncwarp();
        if (go) {
            const int64_t src_row =
                ((int64_t)phys * p.block_size + (t & (p.block_size - 1))) * Hkv + it.h;
            const uint8_t *src = (isv ? vpool : kpool) + src_row * L::kRowBytes;
            const uint32_t dst = stage0 + s * L::kStage + isv * L::kHalf + row * L::kRowStride;
            ptx::bulk_g2s_hint(dst, src, L::kRowBytes, bar, policy);
        }
    };

    for (int s = 0; s < SPW; ++s) {
        Item it;
        int j;
        if (!next_job(it, j))
            break;
        issue(it, j, s);
        ++issued;
    }

    // ---------------- consumer: items in the same order
    SeqCursor cc;
    cursor_reset(cc);
    for (int k = 0;; ++k) {
        const long long g = (long long)blockIdx.x + (long long)k * gridDim.x;
        if (g >= total)
            break;
        const Item it = locate(cc, (int)g, p, lane);
        const int nt = item_tiles(it);
        const T *qhead = static_cast<const T *>(p.q) +
                         ((int64_t)it.b * p.num_q_heads + (int64_t)it.h * G) * D;

        using Math = typename std::conditional<MMA, MmaMath<D, G>, SimtMath<T, D, G>>::type;
        Math math;
        if constexpr (MMA)
            math.begin(reinterpret_cast<const __nv_bfloat16 *>(qhead), p.scale_log2, lane);
        else
            math.begin(qhead, p.scale_log2, lane);
        bool bad = false;

        for (int j = warp; j < nt; j += kWarps) {
            const int s = (int)(consumed % SPW);
            bool ok = false;
            if (consumed < issued) {
                ok = ptx::mbar_wait_bounded(bar0 + 8u * s, (consumed / SPW) & 1u, kWaitLimitNs);
                if (!ok) {
                    aborted = true;
                    if (lane == 0)
                        report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                }
            } else {
                aborted = true;   // job was never issued (only after an abort)
            }
            if ((badmask >> s) & 1u) {
                bad = true;
                badmask &= ~(1u << s);
            }
            if (ok && !bad) {
                const int n = min(kTile, it.t1 - (it.t0 + j * kTile));
                if constexpr (MMA) {
                    const uint32_t ks = stage0 + s * L::kStage;
                    math.tile(ks, ks + L::kHalf, n, p.scale_log2, lane);
                } else {
                    const uint8_t *ks = smem + (warp * SPW + s) * L::kStage;
                    math.tile(ks, ks + L::kHalf, n, scores, lane);
                }
            }
            if (consumed < issued)
                ++consumed;
            // the stage is free again: refill it with the job SPW ahead
            __syncwarp();
            ptx::fence_proxy_async_smem();
            Item nit;
            int nj;
            if (!aborted && next_job(nit, nj)) {
                issue(nit, nj, s);
                ++issued;
            }
        }

        // ---------------- merge the warps' partial softmax states
        float *mrow = merge + warp * L::kMergeFloats;
        math.finish(mrow, lane);
        if (lane == 0)
            mrow[G * D + 2 * G] = bad ? 1.f : 0.f;
        __syncthreads();

        bool anybad = false;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            anybad |= merge[w * L::kMergeFloats + G * D + 2 * G] != 0.f;
        if (threadIdx.x == 0) {
            if (anybad)
                report(p.dev_status, PA_DEV_BAD_BLOCK);
            if (it.ctx_raw != it.ctx && it.part == 0 && it.h == 0)
                report(p.dev_status, PA_DEV_BAD_CONTEXT);
        }
        const int nparts = num_parts(it.ctx, p.partition_size);
        const bool write_final = nparts == 1;
        const bool write_part = nparts > 1 || p.always_partials;
        for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
            const int gq = idx / D;
            const int e = idx - gq * D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w)
                M = fmaxf(M, merge[w * L::kMergeFloats + G * D + gq]);
            float Lsum = 0.f, O = 0.f;
            if (!anybad && M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    const float *row = merge + w * L::kMergeFloats;
                    const float mw = row[G * D + gq];
                    if (mw != -INFINITY) {
                        const float f = ptx::ex2(mw - M);
                        Lsum = fmaf(row[G * D + G + gq], f, Lsum);
                        O = fmaf(row[idx], f, O);
                    }
                }
            }
            const float res = Lsum > 0.f ? O / Lsum : 0.f;
            const int64_t bh = (int64_t)it.b * p.num_q_heads + (int64_t)it.h * G + gq;
            if (write_final)
                store_out<T>(static_cast<T *>(p.out) + bh * D + e, res);
            if (write_part) {
                const int64_t slot = bh * p.max_parts + it.part;
                p.tmp_out[slot * D + e] = res;
                if (e == 0) {
                    const bool empty = anybad || Lsum <= 0.f;
                    p.max_logits[slot] = empty ? -INFINITY : M / kLog2e;
                    p.exp_sums[slot] = empty ? 0.f : Lsum;
                }
            }
        }
        __syncthreads();
    }
}

// =====================================================================
// Split-K reduce: one CTA per (sequence, query head).
// =====================================================================
template <typename T>
__global__ void __launch_bounds__(128) reduce_kernel(const ReduceParams p, int head_dim)
{
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / p.num_q_heads);
    const int ctx = eff_ctx(p.context_lens[b], p.ctx_cap);
    const int n = num_parts(ctx, p.partition_size);
    if (n <= 1)
        return;
    const float *ml = p.max_logits + bh * p.max_parts;
    const float *es = p.exp_sums + bh * p.max_parts;
    float M = -INFINITY;
    for (int i = 0; i < n; ++i)
        M = fmaxf(M, ml[i]);
    for (int e = threadIdx.x; e < head_dim; e += blockDim.x) {
        float Lsum = 0.f, O = 0.f;
        if (M != -INFINITY) {
            for (int i = 0; i < n; ++i) {
                const float l = es[i];
                if (l > 0.f) {
                    const float w = l * ptx::ex2((ml[i] - M) * kLog2e);
                    Lsum += w;
                    O = fmaf(w, p.tmp_out[(bh * p.max_parts + i) * head_dim + e], O);
                }
            }
        }
        store_out<T>(static_cast<T *>(p.out) + bh * head_dim + e, Lsum > 0.f ? O / Lsum : 0.f);
    }
}

}  // namespace pa
