// pa_kernels.cuh -- sm_100a device code of the paged KV-cache decode library.
//
// decode_kernel (persistent, warp-specialised)
//   Work is cut into CTA tiles: 16 consecutive tokens of one sequence for a
//   group of `hpc` KV heads (hpc = min(Hkv, 4)), inside one context partition
//   (the whole context unless the caller asks for fixed-size partitions).  All
//   CTA tiles of the batch form one global sequence ordered by sequence,
//   partition, head group, token.  A "segment" is the run of tiles of one
//   (sequence, partition, head group).  Every CTA owns one contiguous range of
//   that sequence:
//     mode 0 (stream-K): equal ranges.  Every CTA holding a piece of a
//       segment cut by range boundaries publishes the piece's partial softmax
//       state; the last one to do so merges all pieces after its range (all
//       of them share the merge of a segment cut into many pieces).
//       Balanced for any mix of lengths.
//     mode 1: ranges snapped to segment starts, so one CTA finishes every
//       segment it starts (no partials; used without a workspace and for the
//       explicit fixed-partition split-K API).
//   A producer warp streams the CTA's tiles into a ring of SPW shared-memory
//   stages: one TMA tensor-map box brings 16 token rows x d of all hpc heads of
//   K (and one of V), 128-byte swizzled, completing on the stage's "full"
//   mbarrier; block-table entries of the next 32 tiles are fetched in one
//   lane-parallel batch ahead of use; the query rows of a segment come with
//   its first tile.  Consumer warp h (one per head of the group) computes its
//   head's share of each tile and arrives on the stage's "empty" mbarrier.
//
// Tile math (one policy per instantiation)
//   MmaMath   bf16 tensor cores (mma.sync m16n8k16, fp32 accumulate):
//             S = K Q^T with the G query heads of the group as the N = 8
//             columns, then O^T += V^T P^T with P transposed in registers.
//   SimtMath  fp32 FMAs with warp-shuffle dot products (fp32 data; also
//             available for bf16, for comparison).
//   Both keep the online softmax (running max and sum) in fp32, in the log2
//   domain (logits pre-multiplied by log2 e).
//
// reduce_kernel   log-sum-exp merge of fixed-size partitions (explicit API).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <type_traits>

#include "pa.h"
#include "pa_ptx.cuh"

namespace pa {

#ifndef PA_MAX_SPW
#define PA_MAX_SPW 6
#endif

constexpr int kMaxHpc = 4;                  // KV heads per CTA tile, at most
constexpr int kThreads = 32 * (kMaxHpc + 1);// launch bound: consumers + producer
// Over an FP8 cache each KV head has two consumer warps, taking alternate
// tiles (the E4M3 tile math is bound by instruction latency, not by issue)
// (two warpgroups of consumers, then a producer warpgroup of which one warp
// works; the producer warpgroup hands its registers to the consumers)
constexpr int kSubs8 = 2;
constexpr int kThreads8 = 32 * (kMaxHpc * kSubs8 + 4);
constexpr int kRegsLaunch8 = 65536 / kThreads8 / 8 * 8;   // 168 per thread at launch
constexpr int kRegsProducer8 = 72;
constexpr int kRegsConsumer8 = 216;
static_assert(kMaxHpc * kSubs8 * kRegsConsumer8 + 4 * kRegsProducer8 <=
                  (kThreads8 / 32) * kRegsLaunch8,
              "the register split must fit the launch's registers");
constexpr int kMaxSpw = PA_MAX_SPW;         // stages in the ring, at most (FP8 cache)
constexpr int kMaxSpw16 = 4;                // stages in the ring, at most (bf16, f32 caches)
constexpr int kTile = 16;                   // tokens per tile (= MMA M and K)
constexpr int kSmemBudget = 227 * 1024;     // opt-in dynamic shared memory per CTA
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded copy waits: 2 s
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned kFull = 0xffffffffu;

// Shared-memory geometry of one CTA tile, fixed per launch (depends on the
// block size).  A K (or V) region holds 16 token rows of hpc heads as `bpt`
// boxes of `tr` rows; a box is [head][128-byte column][row] with nch = d*elem/128
// columns, i.e. 128-byte line L = (head * nch + column) * tr + row, and
//   byte(box b, line L, 16-byte unit u) = b*box_stride + L*128 + ((u % 8) ^ (L % 8)) * 16
// (the TMA 128-byte swizzle).  Boxes start on 1024-byte boundaries.
struct TileGeo {
    int tr;            // rows per box = min(16, block_size)
    int tr_log2;
    int bpt;           // boxes per tile = 16 / tr
    int hpc;           // KV heads per CTA tile (= consumer warps)
    int head_lines;    // 128-byte lines per head in a box = nch * tr
    int box_stride;    // bytes between boxes
    int kv_bytes;      // bytes of one tile's K (or V) region
    int tps;           // tiles per stage: 1, or 2 over an FP8 cache (K of both, then V of both)
    int q_off;         // offset of the query slot in a stage
    int stage_bytes;   // K + V + query, multiple of 1024
    int spw;           // stages in the ring
    int box_tx;        // bytes one box delivers
    int q_bytes;       // bytes of the query slot payload
    int q_head_bytes;  // query bytes of one KV head (G * d * elem)
};

struct DecodeParams {
    void *out;
    const void *q;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *tmp_out;          // explicit split-K layout [B, Hq, max_parts, d]
    float *max_logits;       // [B, Hq, max_parts]
    float *exp_sums;         // [B, Hq, max_parts]
    float *wpart;            // mode 0: two partial slots per CTA and head
    unsigned long long *counters;  // mode 0: arrivals per cut segment (its first CTA, head), a line each
    int32_t *dev_status;
    int64_t num_blocks;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int max_blocks;
    int block_size;
    int bs_log2;
    int partition_size;      // multiple of 16; >= ctx_cap means the whole context
    int max_parts;
    int ctx_cap;             // lengths above this are invalid
    int mode;                // 0 stream-K, 1 whole segments
    int public_partials;     // mode 1: write tmp_out / max_logits / exp_sums
    int slot_floats;         // floats per partial slot (mode 0)
    int head_groups;         // Hkv / hpc
    uint32_t epoch;          // mode 0: tag of this call's counter values (never 0)
    float scale_log2;
    float out_scale;         // multiplies every output (the V scale of an FP8 cache; else 1)
    uint64_t wait_ns;        // limit of every bounded wait (kWaitLimitNs unless a test sets it)
    int withhold_cta;        // test hook: this CTA's producer withholds its second tile's copy (-1: none)
    TileGeo geo;
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

template <typename T>
__device__ __forceinline__ void store_out(T *dst, float v);
template <>
__device__ __forceinline__ void store_out<float>(float *dst, float v) { *dst = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16 *dst, float v)
{
    *dst = __float2bfloat16_rn(v);
}

// 16 bytes of outputs from VEC = 16 / sizeof(T) floats.
__device__ __forceinline__ void store16(float *dst, const float *x)
{
    *reinterpret_cast<float4 *>(dst) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void store16(__nv_bfloat16 *dst, const float *x)
{
    uint4 u;
    u.x = ptx::pack_bf16x2(x[0], x[1]);
    u.y = ptx::pack_bf16x2(x[2], x[3]);
    u.z = ptx::pack_bf16x2(x[4], x[5]);
    u.w = ptx::pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4 *>(dst) = u;
}

// Four consecutive outputs (16-byte aligned for fp32, 8-byte for bf16).
__device__ __forceinline__ void store4(float *dst, float4 v)
{
    *reinterpret_cast<float4 *>(dst) = v;
}
__device__ __forceinline__ void store4(__nv_bfloat16 *dst, float4 v)
{
    *reinterpret_cast<uint2 *>(dst) = make_uint2(ptx::pack_bf16x2(v.x, v.y), ptx::pack_bf16x2(v.z, v.w));
}

// =====================================================================
// Tile enumeration
// =====================================================================
__device__ __forceinline__ int eff_ctx(int ctx, int cap) { return (ctx < 0 || ctx > cap) ? 0 : ctx; }
__device__ __forceinline__ int num_parts(int ctx, int P) { return ctx <= 0 ? 1 : (ctx + P - 1) / P; }
__device__ __forceinline__ int ntiles(int ctx) { return (ctx + kTile - 1) / kTile; }

constexpr int kMaxChunks = 1024;   // sequences / 32, i.e. batches of up to 32768 sequences

// CTA-cooperative: cbase[c] = global index of the first tile of sequence
// 32 c, for c = 0 .. ceil(B / 32); returns the total tile count.  Must be
// called by every thread of the CTA (contains __syncthreads).
__device__ __forceinline__ int chunk_prefix(const DecodeParams &p, int *cbase)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int nch = (p.num_seqs + 31) >> 5;
    for (int c = warp; c < nch; c += nwarps) {
        const int b = c * 32 + lane;
        int t = b < p.num_seqs ? ntiles(eff_ctx(p.context_lens[b], p.ctx_cap)) * p.head_groups : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            t += __shfl_xor_sync(kFull, t, o);
        if (lane == 0)
            cbase[c + 1] = t;
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        if (lane == 0)
            cbase[0] = 0;
        for (int c0 = 0; c0 < nch; c0 += 32) {
            const int c = c0 + lane;
            int v = c < nch ? cbase[c + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(kFull, v, o);
                if (lane >= o)
                    v += u;
            }
            if (c < nch)
                cbase[c + 1] = carry + v;
            carry += __shfl_sync(kFull, v, 31);
        }
    }
    __syncthreads();
    return cbase[nch];
}

// A window of 32 consecutive sequences with their tile counts, one per lane,
// used to map global tile indices to sequences.
struct SeqWindow {
    int b0;      // first sequence of the window
    int base;    // global index of the first tile of sequence b0
    int cnt;     // this lane's sequence: tiles (head groups * ntiles)
    int incl;    // inclusive prefix of cnt over the window
    int ctx;     // this lane's sequence: effective length
};

__device__ __forceinline__ void window_load(SeqWindow &w, int b0, int base, const DecodeParams &p,
                                            int lane)
{
    w.b0 = b0;
    w.base = base;
    const int b = b0 + lane;
    w.ctx = b < p.num_seqs ? eff_ctx(p.context_lens[b], p.ctx_cap) : 0;
    w.cnt = ntiles(w.ctx) * p.head_groups;
    int incl = w.cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o)
            incl += v;
    }
    w.incl = incl;
}

// Index of the chunk of 32 sequences holding global tile g (binary search
// over the chunk prefix; g must be below the total).
__device__ __forceinline__ int chunk_of(const int *cbase, int nch, int g)
{
    int lo = 0, hi = nch - 1;   // largest c with cbase[c] <= g
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cbase[mid] <= g)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Resolves each lane's global tile index g (ignored where !want) to its
// sequence: b, the global index of the sequence's first tile, and its
// effective length.  The window moves forward by jumping to the chunk of the
// smallest unresolved target, so targets must not precede the window.
// Warp-uniform control flow.
__device__ __forceinline__ void window_find(SeqWindow &w, int g, bool want, int &b, int &seqbase,
                                            int &ctx, const DecodeParams &p, const int *cbase,
                                            int lane)
{
    bool done = !want;
    b = 0;
    seqbase = 0;
    ctx = 0;
    while (true) {
        const int last = w.base + __shfl_sync(kFull, w.incl, 31);
        const bool here = !done && g < last;
        // pos = number of window sequences whose tiles all precede g
        int pos = 0;
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) {
            const int v = __shfl_sync(kFull, w.incl, pos + s - 1);
            if (w.base + v <= g)
                pos += s;
        }
        const int src = pos < 32 ? pos : 31;
        const int incl_at = __shfl_sync(kFull, w.incl, src);
        const int cnt_at = __shfl_sync(kFull, w.cnt, src);
        const int ctx_at = __shfl_sync(kFull, w.ctx, src);
        if (here) {
            b = w.b0 + pos;
            seqbase = w.base + incl_at - cnt_at;
            ctx = ctx_at;
            done = true;
        }
        if (!__any_sync(kFull, !done))
            break;
        if (w.b0 + 32 >= p.num_seqs)   // targets past the last tile: leave them
            break;
        int gmin = done ? INT32_MAX : g;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            gmin = min(gmin, __shfl_xor_sync(kFull, gmin, o));
        const int c = max(chunk_of(cbase, (p.num_seqs + 31) >> 5, gmin), (w.b0 >> 5) + 1);
        window_load(w, c * 32, cbase[c], p, lane);
    }
}

// Tile descriptor (h is the head group); a batch holds 32 consecutive tiles,
// one per lane.
struct TileDesc {
    int b, h, part, j, ns, t0, n, ctx;
    int phys[4];
};

// Descriptor of lane `src` of batch d, to every lane.
__device__ __forceinline__ TileDesc shfl_desc(const TileDesc &d, int src)
{
    TileDesc o;
    o.b = __shfl_sync(kFull, d.b, src);
    o.h = __shfl_sync(kFull, d.h, src);
    o.part = __shfl_sync(kFull, d.part, src);
    o.j = __shfl_sync(kFull, d.j, src);
    o.ns = __shfl_sync(kFull, d.ns, src);
    o.t0 = __shfl_sync(kFull, d.t0, src);
    o.n = __shfl_sync(kFull, d.n, src);
    o.ctx = __shfl_sync(kFull, d.ctx, src);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        o.phys[k] = __shfl_sync(kFull, d.phys[k], src);
    return o;
}

// Fills the descriptors of tiles [base, base + 32) below `end` and starts
// their block-table loads.
__device__ __forceinline__ void fill_batch(TileDesc &d, SeqWindow &w, int base, int end,
                                           const DecodeParams &p, const int *cbase, int lane)
{
    const int g = base + lane;
    const bool want = g < end;
    int b, seqbase, ctx;
    window_find(w, g, want, b, seqbase, ctx, p, cbase, lane);
    d.b = b;
    d.h = 0;
    d.part = 0;
    d.j = 0;
    d.ns = 1;
    d.t0 = 0;
    d.n = 0;
    d.ctx = ctx;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        d.phys[k] = -1;
    if (!want)
        return;
    const int HG = p.head_groups;
    const int nt = ntiles(ctx);
    const int PT = p.partition_size >> 4;             // tiles of a full partition
    const int x = g - seqbase;
    const int nparts = num_parts(ctx, p.partition_size);
    int part = (int)((int64_t)x / ((int64_t)HG * PT));
    if (part > nparts - 1)
        part = nparts - 1;
    const int rem = x - (int)((int64_t)part * HG * PT);
    const int np = min(PT, nt - part * PT);             // tiles of this partition
    d.h = rem / np;
    d.j = rem - d.h * np;
    d.ns = np;
    d.part = part;
    d.t0 = part * p.partition_size + kTile * d.j;
    const int64_t pend = (int64_t)(part + 1) * p.partition_size;
    const int seg_end = pend < ctx ? (int)pend : ctx;
    d.n = min(kTile, seg_end - d.t0);
    const int32_t *row = p.block_tables + (int64_t)b * p.max_blocks;
    const int tr = p.geo.tr;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (k < p.geo.bpt && k * tr < d.n)
            d.phys[k] = row[(d.t0 + k * tr) >> p.bs_log2];
}

// First tile of warp gw's range (T for gw == total_warps).
__device__ __forceinline__ int range_begin(int gw, int total_warps, int T, const DecodeParams &p,
                                           const int *cbase, int lane)
{
    if (gw >= total_warps)
        return T;
    const int x = (int)((int64_t)gw * T / total_warps);
    if (p.mode == 0 || x >= T)
        return x;
    // mode 1: the first segment start at or after x
    SeqWindow w;
    const int c = chunk_of(cbase, (p.num_seqs + 31) >> 5, x);
    window_load(w, c * 32, cbase[c], p, lane);
    TileDesc d;
    fill_batch(d, w, x, x + 1, p, cbase, lane);
    const int j = __shfl_sync(kFull, d.j, 0);
    const int ns = __shfl_sync(kFull, d.ns, 0);
    return j == 0 ? x : x - j + ns;
}

// =====================================================================
// Swizzled addressing of a K or V region
// =====================================================================
// Address of 16-byte unit u of token row t of the head whose lines start at
// line `hline` (= head * head_lines) in a region starting at `reg`.
__device__ __forceinline__ uint32_t kv_addr(uint32_t reg, int hline, int t, int u, const TileGeo &g)
{
    const int box = t >> g.tr_log2;
    const int r = t & (g.tr - 1);
    const uint32_t line = (uint32_t)(hline + (u >> 3) * g.tr + r);
    return reg + (uint32_t)(box * g.box_stride) + line * 128u +
           ((((uint32_t)u & 7u) ^ (line & 7u)) << 4);
}

// Same, for one 16-row box (block size >= 16): the swizzle phase is t & 7.
__device__ __forceinline__ uint32_t kv_addr16(uint32_t reg, int hline, int t, int u)
{
    return reg + (uint32_t)((hline + (u >> 3) * kTile + t) * 128) +
           ((((uint32_t)u & 7u) ^ ((uint32_t)t & 7u)) << 4);
}

template <bool TR16>
__device__ __forceinline__ uint32_t tile_addr(uint32_t reg, int hline, int t, int u,
                                              const TileGeo &g)
{
    if constexpr (TR16)
        return kv_addr16(reg, hline, t, u);
    else
        return kv_addr(reg, hline, t, u, g);
}

// Stores unit u (four accumulator elements) of a published piece whose
// elements have type P: fp32 as they are, bf16 rounded to nearest even.
template <typename P>
__device__ __forceinline__ void put_unit(void *ps, int u, float x, float y, float z, float w)
{
    if constexpr (sizeof(P) == 2)
        reinterpret_cast<uint2 *>(ps)[u] = make_uint2(ptx::pack_bf16x2(x, y), ptx::pack_bf16x2(z, w));
    else
        reinterpret_cast<float4 *>(ps)[u] = make_float4(x, y, z, w);
}

// =====================================================================
// Tile math, bf16 tensor cores (warp-level MMA)
//
// Fragment maps (r = lane / 4, c = lane % 4):
//   S = K Q^T, M = 16 tokens, N = 8 heads (G real), K = d in steps of 16.
//     S frag: s0,s1 = S[tok r][head 2c, 2c+1], s2,s3 = S[tok r+8][...].
//   O^T += V^T P^T, M = 16 d-rows per step k, N = 8 heads, K = 16 tokens.
//     P^T frag from movmatrix of the packed S frag; O^T frag:
//     a0,a1 = O^T[d 16k+r][head 2c, 2c+1], a2,a3 = O^T[d 16k+r+8][...].
// A lane owns heads 2c and 2c+1 in both maps, so the running max, sum and
// rescale of those heads stay in the lane (apart from the max reduction).
// =====================================================================
template <int D, int G, bool TR16>
struct MmaMath {
    static_assert(G <= 8, "group must fit the N = 8 MMA");
    static constexpr int KS = D / 16;

    uint32_t qf[KS][2];
    float acc[KS][4];
    float m[2];
    float l[2];

    // Query fragments from the stage's query slot ([G][D] bf16, row-major).
    __device__ __forceinline__ void begin(const uint8_t *qslot, int lane)
    {
        const int r = lane >> 2, c = lane & 3;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            if (r < G) {
                const uint32_t *qr = reinterpret_cast<const uint32_t *>(qslot + (r * D + 16 * k) * 2);
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

    __device__ __forceinline__ void tile(uint32_t ks, uint32_t vs, int hline, int n,
                                         float scale_log2, const TileGeo &geo, int lane)
    {
        const int r = lane >> 2;
        // ---- S = K Q^T (two accumulation chains)
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        const int krow = lane & 15, khalf = lane >> 4;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            uint32_t a[4];
            ptx::ldsm_x4(tile_addr<TR16>(ks, hline, krow, 2 * k + khalf, geo), a);
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
        const int vrow = (lane & 7) + ((lane >> 4) << 3), vhalf = (lane >> 3) & 1;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            uint32_t a[4];
            ptx::ldsm_x4_trans(tile_addr<TR16>(vs, hline, vrow, 2 * k + vhalf, geo), a);
            ptx::mma_bf16_16816(acc[k], a, b0, b1);
        }
    }

    // Completes the running sums: afterwards every lane holds the sums of its
    // two heads.
    __device__ __forceinline__ void finish()
    {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l[0] += __shfl_xor_sync(kFull, l[0], o);
            l[1] += __shfl_xor_sync(kFull, l[1], o);
        }
    }

    // Published piece layout: the accumulator fragments of the lanes that hold
    // real heads (c < CU), one float4 (acc[k][0..3]) per (k, lane) at unit
    // k * 8 * CU + r * CU + c; then max and sum per head (publish_stats).
    static constexpr int CU = (G + 1) / 2;
    static constexpr int kUnits = KS * 8 * CU;

    template <typename P>
    __device__ __forceinline__ void publish(void *ps, int lane) const
    {
        const int r = lane >> 2, c = lane & 3;
        if (c < CU) {
#pragma unroll
            for (int k = 0; k < KS; ++k)
                put_unit<P>(ps, k * 8 * CU + r * CU + c, acc[k][0], acc[k][1], acc[k][2],
                            acc[k][3]);
        }
    }

    __device__ __forceinline__ void publish_stats(float *st, int lane) const
    {
        const int r = lane >> 2, c = lane & 3;
        if (r == 0 && 2 * c < G) {
            st[2 * c] = m[0];
            st[G + 2 * c] = l[0];
            if (2 * c + 1 < G) {
                st[2 * c + 1] = m[1];
                st[G + 2 * c + 1] = l[1];
            }
        }
    }

    // (head, d) of element j of published unit u (head >= G: padding).
    __device__ __forceinline__ static void unit_coords(int u, int j, int &g, int &d)
    {
        const int k = u / (8 * CU), rem = u - k * 8 * CU;
        const int r = rem / CU, c = rem - r * CU;
        g = 2 * c + (j & 1);
        d = 16 * k + r + 8 * (j >> 1);
    }

    // Writes acc / sum (zeros where `zero` or the sum is 0) to o[head * D + d]
    // as bf16: one reciprocal per head; each 8 x 8 block (d x head) of the
    // normalised accumulators is packed to bf16 pairs and transposed across
    // the warp (movmatrix), so lane (r, c) then holds head r at d = 2c, 2c + 1
    // and stores them as one 4-byte word.
    __device__ __forceinline__ void store_final(__nv_bfloat16 *o, bool zero, int lane) const
    {
        const int r = lane >> 2, c = lane & 3;
        const float i0 = (zero || !(l[0] > 0.f)) ? 0.f : __frcp_rn(l[0]);
        const float i1 = (zero || !(l[1] > 0.f)) ? 0.f : __frcp_rn(l[1]);
        uint32_t *row = reinterpret_cast<uint32_t *>(o + r * D) + c;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const uint32_t lo =
                ptx::movmatrix_trans(ptx::pack_bf16x2(acc[k][0] * i0, acc[k][1] * i1));
            const uint32_t hi =
                ptx::movmatrix_trans(ptx::pack_bf16x2(acc[k][2] * i0, acc[k][3] * i1));
            if (r < G) {
                row[8 * k] = lo;
                row[8 * k + 4] = hi;
            }
        }
    }

    // Calls f(head, d, acc, sum) for every unnormalised accumulator this lane
    // holds (heads < G), and fm(head, max, sum) once per head.
    template <typename F, typename FM>
    __device__ __forceinline__ void for_each(int lane, F f, FM fm) const
    {
        const int r = lane >> 2, c = lane & 3;
        const int h0 = 2 * c, h1 = 2 * c + 1;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int d0 = 16 * k + r;
            if (h0 < G) {
                f(h0, d0, acc[k][0], l[0]);
                f(h0, d0 + 8, acc[k][2], l[0]);
            }
            if (h1 < G) {
                f(h1, d0, acc[k][1], l[1]);
                f(h1, d0 + 8, acc[k][3], l[1]);
            }
        }
        if (r == 0) {
            if (h0 < G)
                fm(h0, m[0], l[0]);
            if (h1 < G)
                fm(h1, m[1], l[1]);
        }
    }
};

// =====================================================================
// Tile math over an E4M3 (FP8) cache: bf16 query and output, one byte per
// K / V element with a per-tensor scale.  The K scale is folded into the
// logit scale, the V scale into the output scale.
//
// Both tile products run on E4M3 tensor cores (mma m16n8k32, fp32
// accumulation) with the K and V codes as they are, so the query and the
// softmax weights must be E4M3 too.  Each query row, scaled by a power of
// two, is split into hi = e4m3(q) and lo = e4m3(q - hi); S = K hi + K lo is
// exact for every element of at least 2^-9 of the row's largest (a bf16
// element has 8 significant bits, hi and lo 4 each).  Each weight, scaled
// by 2^8 (the row's largest is exactly 256), is split into hi = e4m3(x) and
// lo = e4m3(x - hi): hi + lo carries about 8 significant bits, as a bf16
// weight does.  The MMA's reduction index runs over the tile's 16 tokens
// twice, paired once with hi and once with lo, so one MMA adds V (hi + lo).
// The running sums take the same hi + lo values, also scaled by 2^8, so the
// scale cancels in acc / sum (and in the merge of split pieces).
//
// One 16-byte unit of a row holds 16 elements.  ldmatrix reads 8 x 8
// matrices of 16-bit elements, i.e. 8 rows x 16 bytes:
//   S = K Q^T: lane (r, c) receives bytes 4c .. 4c+3 of row (token) r of a
//     unit; four matrices (tokens 0-7 and 8-15 of two consecutive units)
//     are exactly the MMA's A fragment over 32 elements, and the query
//     fragments hold elements 4c .. 4c+3 and 16 + 4c .. 16 + 4c+3 of head r.
//   O^T += V^T P^T (ldmatrix.trans): lane (r, c) receives, from the matrix of
//     tokens 0-7 (m0) and of tokens 8-15 (m1), bytes 2r, 2r+1 of tokens 2c,
//     2c+1.  Byte permutes gather element 2r of tokens 2c, 2c+1, 2c+8, 2c+9
//     (MMA row r, reduction index 4c .. 4c+3) and element 2r+1 (row r + 8);
//     the weight fragment lists the same four tokens, gathered by shuffles
//     from the lanes that computed them.  Accumulator acc[k][0..3] thus holds
//     O[head 2c][16k + 2r], O[head 2c+1][16k + 2r], O[head 2c][16k + 2r + 1],
//     O[head 2c+1][16k + 2r + 1].
// =====================================================================
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t codes)
{
    const __half2_raw h =
        __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(codes & 0xffffu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Two fp32 values to E4M3 codes (round to nearest even, saturating to
// +-448): `lo` in byte 0, `hi` in byte 1.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi)
{
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3) &
           0xffffu;
}

template <int D, int G>
struct MmaMath8 {
    static_assert(G <= 8, "group must fit the N = 8 MMA");
    static constexpr int KS = D / 16;   // 16-byte units per row
    static constexpr int K32 = D / 32;  // 32-element reduction steps
    // Up to four heads: the S product's N = 8 columns hold the hi parts of
    // heads 0-3 (columns 0-3) and their lo parts (columns 4-7), so one MMA
    // per reduction step covers both; lanes (r, c) and (r, c ^ 2) then add
    // their halves and hold the same logits (heads 2 (c & 1), 2 (c & 1) + 1).
    static constexpr bool PACK = G <= 4;

    uint32_t qh[K32][2];   // E4M3 hi parts of sigma * q, this lane's fragment
                           // (PACK: hi for columns 0-3, lo for columns 4-7)
    uint32_t ql[PACK ? 1 : K32][2];   // E4M3 lo parts (not PACK)
    float sf[2];           // logit factor (scale_log2 / sigma) of heads 2c, 2c+1
    float acc[KS][4];
    float m[2];
    float l[2];

    // Query fragments from the segment's query rows ([G][D] bf16, global
    // memory, read through the read-only path).  Head h's row is scaled by a power of two sigma_h (max |sigma_h q| in [128, 256)),
    // then split into hi = e4m3(sigma_h q) and lo = e4m3(sigma_h q - hi):
    // every element of at least 2^-9 max |q| is exactly hi + lo (its 8
    // significant bits land in two 4-bit codes), smaller ones to within
    // 2^-10 / sigma_h.  A non-finite row makes its logits NaN.
    __device__ __forceinline__ void begin(const uint8_t *qrows, int lane, float scale_log2)
    {
        const int r = lane >> 2, c = lane & 3;
        const int hq = PACK ? (r & 3) : r;   // the head of this lane's column
        float x[K32][2][4];
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < K32; ++k)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint2 w = make_uint2(0u, 0u);
                if (hq < G)
                    w = __ldg(reinterpret_cast<const uint2 *>(qrows + (hq * D + 32 * k + 16 * h + 4 * c) * 2));
                x[k][h][0] = ptx::bf16lo_to_f32(w.x);
                x[k][h][1] = ptx::bf16hi_to_f32(w.x);
                x[k][h][2] = ptx::bf16lo_to_f32(w.y);
                x[k][h][3] = ptx::bf16hi_to_f32(w.y);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    amax = fmaxf(amax, fabsf(x[k][h][i]));
            }
        amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
        // sigma = 2^(7 - floor(log2 amax)), from the exponent field
        const int ef = (int)((__float_as_uint(amax) >> 23) & 0xffu);
        const float sigma = __uint_as_float((uint32_t)min(254, 261 - ef) << 23);
        const float fac = amax <= 3.4028235e38f ? scale_log2 / sigma : __int_as_float(0x7fc00000);
#pragma unroll
        for (int k = 0; k < K32; ++k)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float y0 = x[k][h][0] * sigma, y1 = x[k][h][1] * sigma;
                const float y2 = x[k][h][2] * sigma, y3 = x[k][h][3] * sigma;
                const uint32_t h01 = f32x2_to_e4m3x2(y0, y1), h23 = f32x2_to_e4m3x2(y2, y3);
                const uint32_t f01 = e4m3x2_to_f16x2(h01), f23 = e4m3x2_to_f16x2(h23);
                const uint32_t l01 = f32x2_to_e4m3x2(y0 - ptx::f16lo_to_f32(f01),
                                                     y1 - ptx::f16hi_to_f32(f01));
                const uint32_t l23 = f32x2_to_e4m3x2(y2 - ptx::f16lo_to_f32(f23),
                                                     y3 - ptx::f16hi_to_f32(f23));
                if constexpr (PACK) {
                    qh[k][h] = r < 4 ? h01 | (h23 << 16) : l01 | (l23 << 16);
                } else {
                    qh[k][h] = h01 | (h23 << 16);
                    ql[k][h] = l01 | (l23 << 16);
                }
            }
        // lane (r, c) scales the logits of heads 2c', 2c'+1 (c' = c, or c & 1
        // with PACK), whose factors the lanes of rows 2c', 2c'+1 computed
        const int cs = PACK ? (c & 1) : c;
        sf[0] = __shfl_sync(kFull, fac, 8 * cs);
        sf[1] = __shfl_sync(kFull, fac, 8 * cs + 4);
#pragma unroll
        for (int k = 0; k < KS; ++k)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[k][i] = 0.f;
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
    }

    __device__ __forceinline__ void tile(uint32_t ks, uint32_t vs, int hline, int n,
                                         float scale_log2, const TileGeo &geo, int lane)
    {
        const int r = lane >> 2;
        const int row = (lane & 7) + (((lane >> 3) & 1) << 3), half = lane >> 4;
        // ---- S = K (hi + lo)^T on E4M3 tensor cores, four accumulation chains
        float c4[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            c4[j][0] = c4[j][1] = c4[j][2] = c4[j][3] = 0.f;
        float s[4];
        if constexpr (PACK) {
#pragma unroll
            for (int k = 0; k < K32; ++k) {
                uint32_t a[4];
                ptx::ldsm_x4(kv_addr16(ks, hline, row, 2 * k + half), a);
                ptx::mma_e4m3_16832(c4[k & 3], a, qh[k][0], qh[k][1]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float h = (c4[0][i] + c4[1][i]) + (c4[2][i] + c4[3][i]);
                // hi (columns 0-3) plus lo (columns 4-7): the same sum in both lanes
                s[i] = (h + __shfl_xor_sync(kFull, h, 2)) * sf[i & 1];
            }
        } else {
#pragma unroll
            for (int k = 0; k < K32; ++k) {
                uint32_t a[4];
                ptx::ldsm_x4(kv_addr16(ks, hline, row, 2 * k + half), a);
                ptx::mma_e4m3_16832(c4[2 * (k & 1)], a, qh[k][0], qh[k][1]);
                ptx::mma_e4m3_16832(c4[2 * (k & 1) + 1], a, ql[k][0], ql[k][1]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                s[i] = ((c4[0][i] + c4[1][i]) + (c4[2][i] + c4[3][i])) * sf[i & 1];
        }
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
        // weights x = 2^8 p: exponents against the new max less 8
        const float rf0 = (mn0 == -INFINITY ? 0.f : mn0) - 8.f;
        const float rf1 = (mn1 == -INFINITY ? 0.f : mn1) - 8.f;
        m[0] = mn0;
        m[1] = mn1;
        const float x0 = ptx::ex2(s[0] - rf0), x1 = ptx::ex2(s[1] - rf1);
        const float x2 = ptx::ex2(s[2] - rf0), x3 = ptx::ex2(s[3] - rf1);
        // hi = e4m3(x), lo = e4m3(x - hi); x - hi is exact in fp32
        const uint32_t h01 = f32x2_to_e4m3x2(x0, x1), h23 = f32x2_to_e4m3x2(x2, x3);
        const uint32_t hf01 = e4m3x2_to_f16x2(h01), hf23 = e4m3x2_to_f16x2(h23);
        const float y0 = ptx::f16lo_to_f32(hf01), y1 = ptx::f16hi_to_f32(hf01);
        const float y2 = ptx::f16lo_to_f32(hf23), y3 = ptx::f16hi_to_f32(hf23);
        const uint32_t l01 = f32x2_to_e4m3x2(x0 - y0, x1 - y1);
        const uint32_t l23 = f32x2_to_e4m3x2(x2 - y2, x3 - y3);
        const uint32_t lf01 = e4m3x2_to_f16x2(l01), lf23 = e4m3x2_to_f16x2(l23);
        // the sums use the same hi + lo as the MMA
        l[0] = l[0] * al0 + ((y0 + ptx::f16lo_to_f32(lf01)) + (y2 + ptx::f16lo_to_f32(lf23)));
        l[1] = l[1] * al1 + ((y1 + ptx::f16hi_to_f32(lf01)) + (y3 + ptx::f16hi_to_f32(lf23)));
        if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                acc[k][0] *= al0;
                acc[k][1] *= al1;
                acc[k][2] *= al0;
                acc[k][3] *= al1;
            }
        }
        // lane (r, c) holds the weights of tokens r, r + 8 for heads 2c, 2c+1:
        // bytes [x(r, 2c), x(r, 2c+1), x(r+8, 2c), x(r+8, 2c+1)].  The weight
        // fragment of lane (r, c) wants head r at tokens 2c, 2c+1, 2c+8, 2c+9,
        // held by lanes (2c, r/2) and (2c+1, r/2), byte r%2 and 2 + r%2.
        const uint32_t whi = h01 | (h23 << 16), wlo = l01 | (l23 << 16);
        const int srcA = 8 * (lane & 3) + (r >> 1);
        const uint32_t sel = (r & 1) ? 0x7351u : 0x6240u;
        const uint32_t b0 =
            ptx::prmt(__shfl_sync(kFull, whi, srcA), __shfl_sync(kFull, whi, srcA + 4), sel);
        const uint32_t b1 =
            ptx::prmt(__shfl_sync(kFull, wlo, srcA), __shfl_sync(kFull, wlo, srcA + 4), sel);
        // ---- O^T += V^T (hi + lo)^T, two 16-element units per ldmatrix
#pragma unroll
        for (int k2 = 0; k2 < KS / 2; ++k2) {
            uint32_t a[4];
            ptx::ldsm_x4_trans(kv_addr16(vs, hline, row, 2 * k2 + half), a);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t e0 = ptx::prmt(a[2 * u], a[2 * u + 1], 0x6420u);   // element 2r
                const uint32_t e1 = ptx::prmt(a[2 * u], a[2 * u + 1], 0x7531u);   // element 2r+1
                const uint32_t f[4] = {e0, e1, e0, e1};
                ptx::mma_e4m3_16832(acc[2 * k2 + u], f, b0, b1);
            }
        }
    }

    __device__ __forceinline__ void finish()
    {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l[0] += __shfl_xor_sync(kFull, l[0], o);
            l[1] += __shfl_xor_sync(kFull, l[1], o);
        }
    }

    // Hands this warp's partial state (before finish) to the head's other
    // warp: accumulator element e (= 4 k + j) of lane x at kx[32 e + x] for
    // e < 2 KS (the head's K lines of the stage just used) and at
    // vx[32 (e - 2 KS) + x] for the rest (its V lines); max, sum and bad mark
    // at st[32 i + x].
    __device__ __forceinline__ void save(float *kx, float *vx, float *st, bool bad,
                                         int lane) const
    {
#pragma unroll
        for (int k = 0; k < KS; ++k)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = 4 * k + j;
                if (e < 2 * KS)
                    kx[32 * e + lane] = acc[k][j];
                else
                    vx[32 * (e - 2 * KS) + lane] = acc[k][j];
            }
        st[lane] = m[0];
        st[32 + lane] = m[1];
        st[64 + lane] = l[0];
        st[96 + lane] = l[1];
        st[128 + lane] = bad ? 1.f : 0.f;
    }

    // Adds the other warp's partial state (same lane layout, disjoint tiles
    // of the segment; placed as `save` does): the log-sum-exp combination of
    // two online-softmax states.  Returns its bad mark.
    __device__ __forceinline__ bool absorb(const float *kx, const float *vx, const float *st,
                                           int lane)
    {
        const float mp0 = st[lane], mp1 = st[32 + lane];
        const float mn0 = fmaxf(m[0], mp0), mn1 = fmaxf(m[1], mp1);
        const float a0 = mn0 == -INFINITY ? 1.f : ptx::ex2(m[0] - mn0);
        const float a1 = mn1 == -INFINITY ? 1.f : ptx::ex2(m[1] - mn1);
        const float b0 = mn0 == -INFINITY ? 1.f : ptx::ex2(mp0 - mn0);
        const float b1 = mn1 == -INFINITY ? 1.f : ptx::ex2(mp1 - mn1);
#pragma unroll
        for (int k = 0; k < KS; ++k)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = 4 * k + j;
                const float o = e < 2 * KS ? kx[32 * e + lane] : vx[32 * (e - 2 * KS) + lane];
                acc[k][j] = acc[k][j] * ((j & 1) ? a1 : a0) + o * ((j & 1) ? b1 : b0);
            }
        l[0] = l[0] * a0 + st[64 + lane] * b0;
        l[1] = l[1] * a1 + st[96 + lane] * b1;
        m[0] = mn0;
        m[1] = mn1;
        return st[128 + lane] != 0.f;
    }

    // Published piece layout: as MmaMath (one float4 acc[k][0..3] per unit
    // k * 8 * CU + r * CU + c), with this layout's element coordinates.
    static constexpr int CU = (G + 1) / 2;
    static constexpr int kUnits = KS * 8 * CU;

    template <typename P>
    __device__ __forceinline__ void publish(void *ps, int lane) const
    {
        const int r = lane >> 2, c = lane & 3;
        if (c < CU) {
#pragma unroll
            for (int k = 0; k < KS; ++k)
                put_unit<P>(ps, k * 8 * CU + r * CU + c, acc[k][0], acc[k][1], acc[k][2],
                            acc[k][3]);
        }
    }

    __device__ __forceinline__ void publish_stats(float *st, int lane) const
    {
        const int r = lane >> 2, c = lane & 3;
        if (r == 0 && 2 * c < G) {
            st[2 * c] = m[0];
            st[G + 2 * c] = l[0];
            if (2 * c + 1 < G) {
                st[2 * c + 1] = m[1];
                st[G + 2 * c + 1] = l[1];
            }
        }
    }

    __device__ __forceinline__ static void unit_coords(int u, int j, int &g, int &d)
    {
        const int k = u / (8 * CU), rem = u - k * 8 * CU;
        const int r = rem / CU, c = rem - r * CU;
        g = 2 * c + (j & 1);
        d = 16 * k + 2 * r + (j >> 1);
    }

    // Writes out_scale * acc / sum (zeros where `zero` or the sum is 0) to
    // o[head * D + d] as bf16: lane (r, c) holds two consecutive d of heads
    // 2c and 2c + 1 and stores each pair as one 4-byte word.
    __device__ __forceinline__ void store_final(__nv_bfloat16 *o, bool zero, float out_scale,
                                                int lane) const
    {
        const int r = lane >> 2, c = lane & 3;
        const float i0 = (zero || !(l[0] > 0.f)) ? 0.f : out_scale * __frcp_rn(l[0]);
        const float i1 = (zero || !(l[1] > 0.f)) ? 0.f : out_scale * __frcp_rn(l[1]);
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            if (2 * c < G)
                *reinterpret_cast<uint32_t *>(o + (2 * c) * D + 16 * k + 2 * r) =
                    ptx::pack_bf16x2(acc[k][0] * i0, acc[k][2] * i0);
            if (2 * c + 1 < G)
                *reinterpret_cast<uint32_t *>(o + (2 * c + 1) * D + 16 * k + 2 * r) =
                    ptx::pack_bf16x2(acc[k][1] * i1, acc[k][3] * i1);
        }
    }

    template <typename F, typename FM>
    __device__ __forceinline__ void for_each(int lane, F f, FM fm) const
    {
        const int r = lane >> 2, c = lane & 3;
        const int h0 = 2 * c, h1 = 2 * c + 1;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int d0 = 16 * k + 2 * r;
            if (h0 < G) {
                f(h0, d0, acc[k][0], l[0]);
                f(h0, d0 + 1, acc[k][2], l[0]);
            }
            if (h1 < G) {
                f(h1, d0, acc[k][1], l[1]);
                f(h1, d0 + 1, acc[k][3], l[1]);
            }
        }
        if (r == 0) {
            if (h0 < G)
                fm(h0, m[0], l[0]);
            if (h1 < G)
                fm(h1, m[1], l[1]);
        }
    }
};

// =====================================================================
// Tile math, CUDA cores
// =====================================================================
template <typename T, int D, int G, bool TR16>
struct SimtMath {
    static constexpr int VEC = 16 / (int)sizeof(T);   // elements per 16-byte unit
    static constexpr int NU = D / VEC;                 // units per row
    static constexpr int LPR = NU < 32 ? NU : 32;      // lanes per row
    static constexpr int RPI = 32 / LPR;               // rows side by side
    static constexpr int UPL = NU / LPR;               // units per lane
    static constexpr int NE = UPL * VEC;               // elements per lane
    static constexpr int RPL = kTile / RPI;            // rows per lane per tile

    float q[G][NE];
    float acc[G][NE];
    float m[G];   // running max, log2 domain (warp-uniform)
    float l[G];   // running sum over this lane's rows

    __device__ __forceinline__ static void cvt(const uint4 u, float (&x)[VEC])
    {
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

    __device__ __forceinline__ static uint4 lds128(uint32_t addr)
    {
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(addr));
        return v;
    }

    __device__ __forceinline__ void begin(const uint8_t *qslot, int lane, float scale_log2)
    {
        const int li = lane % LPR;
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int c = 0; c < UPL; ++c) {
                float x[VEC];
                cvt(*reinterpret_cast<const uint4 *>(qslot + (g * D + (c * LPR + li) * VEC) *
                                                                 (int)sizeof(T)),
                    x);
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

    __device__ __forceinline__ void tile(uint32_t ks, uint32_t vs, int hline, int n,
                                         float *scores, const TileGeo &geo, int lane)
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
            for (int c = 0; c < UPL; ++c) {
                float k[VEC];
                cvt(lds128(tile_addr<TR16>(ks, hline, r, c * LPR + li, geo)), k);
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
                for (int c = 0; c < UPL; ++c) {
                    float v[VEC];
                    cvt(lds128(tile_addr<TR16>(vs, hline, r, c * LPR + li, geo)), v);
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

    // Sums acc and l over the row groups: afterwards lanes of row group 0 hold
    // the accumulator totals and every lane holds the sums.
    __device__ __forceinline__ void finish()
    {
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
    }

    // Published piece layout: acc in [G][D] order, float4 units; then max and
    // sum per head (publish_stats).
    static constexpr int kUnits = G * D / 4;

    template <typename P>
    __device__ __forceinline__ void publish(void *ps, int lane) const
    {
        const int li = lane % LPR;
        if (lane / LPR != 0)
            return;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int c = 0; c < UPL; ++c)
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q)
                    put_unit<P>(ps, (g * D + (c * LPR + li) * VEC + 4 * q) / 4,
                                acc[g][c * VEC + 4 * q], acc[g][c * VEC + 4 * q + 1],
                                acc[g][c * VEC + 4 * q + 2], acc[g][c * VEC + 4 * q + 3]);
    }

    __device__ __forceinline__ void publish_stats(float *st, int lane) const
    {
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                st[g] = m[g];
                st[G + g] = l[g];
            }
        }
    }

    __device__ __forceinline__ static void unit_coords(int u, int j, int &g, int &d)
    {
        g = 4 * u / D;
        d = 4 * u - g * D + j;
    }

    // Writes acc / sum (zeros where `zero` or the sum is 0) to o[g * D + d],
    // VEC consecutive d per 16-byte store; lanes of row group 0 hold them.
    __device__ __forceinline__ void store_final(T *o, bool zero, int lane) const
    {
        const int li = lane % LPR;
        if (lane / LPR != 0)
            return;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float inv = (zero || !(l[g] > 0.f)) ? 0.f : __frcp_rn(l[g]);
#pragma unroll
            for (int c = 0; c < UPL; ++c) {
                float x[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v)
                    x[v] = acc[g][c * VEC + v] * inv;
                store16(o + g * D + (c * LPR + li) * VEC, x);
            }
        }
    }

    template <typename F, typename FM>
    __device__ __forceinline__ void for_each(int lane, F f, FM fm) const
    {
        const int li = lane % LPR;
        const int rg = lane / LPR;
        if (rg == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int c = 0; c < UPL; ++c)
#pragma unroll
                    for (int v = 0; v < VEC; ++v)
                        f(g, (c * LPR + li) * VEC + v, acc[g][c * VEC + v], l[g]);
        }
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g)
                fm(g, m[g], l[g]);
        }
    }
};

// Bytes of one head's exchange area (FP8 cache, two warps per head): the
// max, sum and bad mark of the partial softmax state one warp hands the
// other at a segment end, one float per lane and item, then a "full" and a
// "free" mbarrier.  (The accumulator goes through the stage the handing
// warp used last, which it keeps until the state has been read.)
__host__ __device__ constexpr int exchange_bytes(int D)
{
    return (32 * 5 * 4 + 16 + 127) / 128 * 128 + 0 * D;
}

// Two mbarriers per consumer warp for the bulk copies of its merges.
constexpr int kMergeBarBytes = 16 * kMaxHpc * kSubs8;

// Offset of the merge barriers (then the exchange areas) from the end of
// the stages.
__host__ __device__ constexpr int exchange_off(int G)
{
    return (64 * kMaxSpw + kMaxHpc * kTile * G * 4 + 4 * (kMaxChunks + 1) + 16 + 127) / 128 * 128;
}

// Bytes of the decode kernel's dynamic shared memory besides the stages:
// alignment slack, full and empty barriers, per-stage tile metadata, the
// CUDA-core math's score rows, the chunk prefix of the tile counts, and
// (FP8 cache) the heads' exchange areas.
__host__ __device__ constexpr int decode_smem_fixed(int G, int D = 0, bool kv8 = false)
{
    return 1024 + exchange_off(G) + kMergeBarBytes + (kv8 ? kMaxHpc * exchange_bytes(D) : 0);
}

// Tile metadata the producer warp hands to the consumer warps with a stage.
struct StageMeta {
    int b, hg, part, j, ns, n, ctx, bad;   // of the stage's first tile (bad: either tile)
    int k;                                 // the first tile's offset in the CTA's range
    int nt;                                // tiles in the stage (1 or 2, same segment)
    int n1;                                // tokens of the second tile
    int end;                               // no tiles: the range is done (FP8 ring)
};

// Index of the CTA whose range [R(x), R(x + 1)), R(x) = x T / C, holds tile t.
__device__ __forceinline__ int cta_of(int t, int C, int T)
{
    return (int)((((int64_t)t + 1) * C - 1) / T);
}

// Slot of the piece that CTA x holds of a cut segment: 2x + 1 when the
// segment starts inside the CTA's range (its first piece), 2x otherwise (a
// later piece, met at the start of the range).  Times hpc, plus the head.
__device__ __forceinline__ int piece_slot(int x, bool first, int hpc, int hl)
{
    return (2 * x + (first ? 1 : 0)) * hpc + hl;
}

// 64-bit words per 128-byte line: every arrival counter sits on a line of
// its own, so that the atomics of one segment do not queue behind another's.
constexpr int kLineWords = 16;

__device__ __forceinline__ unsigned long long *counter_of(const DecodeParams &p, int x, int hl)
{
    return p.counters + ((int64_t)x * p.geo.hpc + hl) * kLineWords;
}

// Offset (floats) of a published piece's max / sum / bad mark: after the
// accumulator units of either tile math (the tensor-core layout pads an odd
// group to an even one).
__host__ __device__ constexpr int piece_stats_off(int D, int G) { return 2 * D * ((G + 1) / 2); }

// The same, in floats, for a piece whose accumulator elements have `bytes`
// bytes (4: fp32, 2: bf16); the stats follow the accumulator directly.
__host__ __device__ constexpr int piece_stats_off(int D, int G, int bytes)
{
    return piece_stats_off(D, G) * bytes / 4;
}

// A published piece's stats (max [G], sum [G], bad mark) in float4 units.
__host__ __device__ constexpr int stats_units(int G) { return (2 * G + 1 + 3) / 4; }

// Bytes of per-warp shared scratch a merge of a cut segment of up to np
// pieces needs: np stats blocks and np x G weights (rounded to 128 bytes),
// then two copy buffers of at least one piece's accumulator each.
__host__ __device__ constexpr int64_t merge_header_bytes(int G, int64_t np)
{
    return (4 * (4 * np * stats_units(G) + np * G) + 127) / 128 * 128;
}
__host__ __device__ constexpr int64_t merge_scratch_bytes(int G, int D, int64_t np)
{
    return merge_header_bytes(G, np) + 2 * 4 * (int64_t)piece_stats_off(D, G);
}

// Counts one more arrival at a cut segment's counter for this call and
// returns the arrivals so far including this one (0 if the count could not
// be taken, which cannot happen while fewer than 2^20 pieces race).
//
// The high half of a counter word holds the epoch of the call that counts
// in it; a word with another epoch counts as zero.  Nothing needs to be
// initialised and no arrival waits for another CTA:
//   - the CTA owning the counter raises it to (epoch, 0) with an atomic
//     maximum when it starts, which leaves a count of this call untouched
//     (epochs of one process increase);
//   - an arrival adds 1 with an acquire-release atomic add; if the word it
//     added to carried another epoch, it restarts the count as (epoch, 1)
//     with a compare-and-swap on the value its add left.  A restart erases
//     the adds other arrivals made to the stale word: each of them sees its
//     own swap fail on a word of this epoch and adds again.
// Every arrival is therefore counted once in this epoch.  The add (or the
// swap) releases the caller's piece, stored before it, and the last arrival
// acquires every earlier one.
__device__ __forceinline__ int segment_arrive(unsigned long long *c, uint32_t epoch)
{
    unsigned long long old = ptx::atom_add_acq_rel_gpu(c, 1ull);
    if ((uint32_t)(old >> 32) == epoch)
        return (int)(old & 0xffffffffu) + 1;
    const unsigned long long mine = ((unsigned long long)epoch << 32) | 1ull;
    unsigned long long cur = old + 1;
    for (uint32_t i = 0; i < (1u << 20); ++i) {
        const unsigned long long prev = ptx::atom_cas_acq_rel_gpu(c, cur, mine);
        if (prev == cur)
            return 1;
        if ((uint32_t)(prev >> 32) == epoch) {
            // another arrival restarted the count, erasing this one's add
            old = ptx::atom_add_acq_rel_gpu(c, 1ull);
            if ((uint32_t)(old >> 32) == epoch)
                return (int)(old & 0xffffffffu) + 1;
            cur = old + 1;
        } else {
            cur = prev;   // more adds to the stale word since: swap that value
        }
    }
    return 0;
}

// Weight of head g among a lane's G per-head values (G is small: the
// selection unrolls into compares, keeping the values in registers).
template <int G>
__device__ __forceinline__ float pick(const float (&v)[G], int g)
{
    float r = 0.f;
#pragma unroll
    for (int k = 0; k < G; ++k)
        r = (k == g) ? v[k] : r;
    return r;
}

// Per-head maxima, sums and weights of a cut segment's pieces from their
// stats in shared memory (piece i's max [G] and sum [G] at st[i * stride]),
// by a whole warp: lane i handles
// pieces i, i + 32, ...; the butterflies run in a fixed order, so the result
// does not depend on timing.  Leaves w_i = 2^(m_i - M) / L * out_scale for
// the pieces a lane handles in wl[G] (first piece only) and, with `w`, for
// every piece in w[np][G].
template <int G>
__device__ __forceinline__ void piece_weights(const float *st, int stride, int np, float out_scale,
                                              float *w, float (&wl)[G], int lane)
{
    float M[G], L[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        M[g] = -INFINITY;
        L[g] = 0.f;
    }
    for (int i = lane; i < np; i += 32)
#pragma unroll
        for (int g = 0; g < G; ++g)
            M[g] = fmaxf(M[g], st[i * stride + g]);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            M[g] = fmaxf(M[g], __shfl_xor_sync(kFull, M[g], o));
    for (int i = lane; i < np; i += 32)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mi = st[i * stride + g];
            if (M[g] != -INFINITY && mi != -INFINITY)
                L[g] = fmaf(st[i * stride + G + g], ptx::ex2(mi - M[g]), L[g]);
        }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            L[g] += __shfl_xor_sync(kFull, L[g], o);
#pragma unroll
    for (int g = 0; g < G; ++g)
        wl[g] = 0.f;
    for (int i = lane; i < np; i += 32)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mi = st[i * stride + g];
            // out_scale (1 unless the cache is FP8) multiplies the weights exactly
            const float wi = (mi == -INFINITY || !(L[g] > 0.f))
                                 ? 0.f
                                 : ptx::ex2(mi - M[g]) / L[g] * out_scale;
            if (w)
                w[i * G + g] = wi;
            if (i == lane)
                wl[g] = wi;
        }
}

// Merge of a segment cut into np pieces (CTAs x0 .. x0 + np - 1), for head
// hl of the group, by the warp whose arrival completed the segment's count,
// after its range.  The result is the log-sum-exp combination of the pieces'
// partial softmax states (max m_i, sum l_i, accumulator a_i, log2 domain):
//     M = max_i m_i,   L = sum_i l_i 2^(m_i - M),   o = sum_i a_i 2^(m_i - M) / L,
// the identity the split-K reduction uses.  The pieces' stats go through
// shared memory (`scratch`, `cap` bytes, at least merge_scratch_bytes); the
// accumulators come into two shared buffers by bulk copies (H pieces per
// copy, the next copy in flight while a buffer is summed; two mbarriers at
// `bars`, their phase parities in `phase`), and the weighted sums run in
// piece order, so that the result does not depend on timing.
template <typename T, int D, int G, typename Math>
__device__ __forceinline__ void merge_last(const DecodeParams &p, int x0, int np, int64_t bh0,
                                           int hl, uint8_t *scratch, int cap, uint32_t bars,
                                           uint32_t &phase, int lane)
{
    constexpr int U = Math::kUnits;
    constexpr int UL = (U + 31) / 32;
    constexpr int SO = piece_stats_off(D, G, (int)sizeof(T));
    constexpr int UB = SO * 4;   // bytes of a piece's accumulator region (U units, padded)
    constexpr int SU = stats_units(G);
    const int hpc = p.geo.hpc;
    T *out = static_cast<T *>(p.out) + bh0 * D;
    float *stats = reinterpret_cast<float *>(scratch);   // [np][SU] float4
    float *w = stats + 4 * np * SU;                      // [np][G]
    constexpr int PB = UB + 16 * SU;   // a piece: accumulator, then its stats
    // one copy of every whole piece when they all fit; otherwise the stats
    // first, then the accumulators in batches of H, double buffered
    const int whdr = (np * G * 4 + 127) & ~127;
    const bool one_shot = whdr + np * PB <= cap;
    uint8_t *bufs = one_shot ? scratch + whdr : scratch + merge_header_bytes(G, np);
    if (one_shot)
        w = reinterpret_cast<float *>(scratch);
    const int H = one_shot ? np : max(1, min(np, (cap - (int)merge_header_bytes(G, np)) / (2 * UB)));
    const int CB = one_shot ? PB : UB;   // bytes copied per piece
    auto src = [&](int i) {
        return p.wpart + (int64_t)piece_slot(x0 + i, i == 0, hpc, hl) * p.slot_floats;
    };
    auto zero_out = [&]() {
#pragma unroll
        for (int t = 0; t < UL; ++t) {
            const int e = lane + 32 * t;
            if (e < U)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    int g, d;
                    Math::unit_coords(e, j, g, d);
                    if (g < G)
                        store_out<T>(out + g * D + d, 0.f);
                }
        }
        __syncwarp();
    };
    // the copies read the pieces (published by generic stores, acquired by
    // the arrival count) and overwrite shared memory this warp's generic
    // accesses used before: order both before them
    ptx::fence_proxy_async_all();
    __syncwarp();
    const int nb = (np + H - 1) / H;
    auto issue = [&](int bt) {
        if (lane == 0) {
            const int i0 = bt * H, n = min(H, np - i0);
            const uint32_t bar = bars + 8u * (uint32_t)(bt & 1);
            ptx::mbar_arrive_expect_tx(bar, (uint32_t)(n * CB));
            for (int i = 0; i < n; ++i)
                ptx::bulk_g2s(ptx::smem_u32(bufs + ((bt & 1) * H + i) * CB), src(i0 + i),
                              (uint32_t)CB, bar);
        }
        __syncwarp();
    };
    bool bad = false;
    float wl[G];
    if (one_shot) {
        issue(0);
        if (!ptx::mbar_wait_bounded(bars, phase & 1u, p.wait_ns)) {
            phase ^= 1u;
            if (lane == 0)
                report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
            zero_out();
            return;
        }
        phase ^= 1u;
        const float *st0 = reinterpret_cast<const float *>(bufs + UB);
        for (int i = lane; i < np; i += 32)
            bad |= st0[i * (PB / 4) + 2 * G] != 0.f;
        bad = __any_sync(kFull, bad);
        if (!bad)
            piece_weights<G>(st0, PB / 4, np, p.out_scale, w, wl, lane);
        __syncwarp();
    } else {
        // the stats go first: they decide the weights, the copies only the sums
        for (int i = lane; i < np; i += 32) {
            const float4 *s4 = reinterpret_cast<const float4 *>(src(i) + SO);
#pragma unroll
            for (int u = 0; u < SU; ++u)
                reinterpret_cast<float4 *>(stats)[i * SU + u] = __ldcg(s4 + u);
            bad |= stats[i * 4 * SU + 2 * G] != 0.f;
        }
        bad = __any_sync(kFull, bad);
        __syncwarp();
        issue(0);
        if (nb > 1)
            issue(1);
        if (!bad)
            piece_weights<G>(stats, 4 * SU, np, p.out_scale, w, wl, lane);
        __syncwarp();
    }
    float o[UL][4];
#pragma unroll
    for (int t = 0; t < UL; ++t)
        o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    for (int bt = 0; bt < nb; ++bt) {
        const uint32_t bar = bars + 8u * (uint32_t)(bt & 1);
        bool ok = true;
        if (!one_shot) {
            ok = ptx::mbar_wait_bounded(bar, (phase >> (bt & 1)) & 1u, p.wait_ns);
            phase ^= 1u << (bt & 1);
        }
        if (!ok || bad) {
            // let the other buffer's copy land (bounded) before leaving
            if (!one_shot && bt + 1 < nb) {
                ptx::mbar_wait_bounded(bars + 8u * (uint32_t)((bt + 1) & 1),
                                       (phase >> ((bt + 1) & 1)) & 1u, p.wait_ns);
                phase ^= 1u << ((bt + 1) & 1);
            }
            if (lane == 0)
                report(p.dev_status, ok ? PA_DEV_BAD_BLOCK : PA_DEV_WAIT_TIMEOUT);
            zero_out();
            return;
        }
        const int i0 = bt * H, n = min(H, np - i0);
        for (int i = 0; i < n; ++i) {
            float wp[G];
#pragma unroll
            for (int g = 0; g < G; ++g)
                wp[g] = w[(i0 + i) * G + g];
            const uint8_t *bp = bufs + ((bt & 1) * H + i) * CB;
#pragma unroll
            for (int t = 0; t < UL; ++t) {
                const int e = lane + 32 * t;
                if (e < U) {
                    float vv[4];
                    if constexpr (sizeof(T) == 2) {
                        const uint2 v = reinterpret_cast<const uint2 *>(bp)[e];
                        vv[0] = ptx::bf16lo_to_f32(v.x);
                        vv[1] = ptx::bf16hi_to_f32(v.x);
                        vv[2] = ptx::bf16lo_to_f32(v.y);
                        vv[3] = ptx::bf16hi_to_f32(v.y);
                    } else {
                        const float4 v = reinterpret_cast<const float4 *>(bp)[e];
                        vv[0] = v.x;
                        vv[1] = v.y;
                        vv[2] = v.z;
                        vv[3] = v.w;
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        int g, d;
                        Math::unit_coords(e, j, g, d);
                        o[t][j] = fmaf(pick<G>(wp, g), vv[j], o[t][j]);
                    }
                }
            }
        }
        if (bt + 2 < nb) {
            // this buffer's generic reads come before the next copy into it
            ptx::fence_proxy_async_smem();
            __syncwarp();
            issue(bt + 2);
        }
    }
#pragma unroll
    for (int t = 0; t < UL; ++t) {
        const int e = lane + 32 * t;
        if (e < U)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int g, d;
                Math::unit_coords(e, j, g, d);
                if (g < G)
                    store_out<T>(out + g * D + d, o[t][j]);
            }
    }
    __syncwarp();
}

// Sequence, head group, index in the segment and the segment's tiles of
// global tile g (no block-table loads).  Warp-uniform; g below the total.
__device__ __forceinline__ void tile_segment(int g, const DecodeParams &p, const int *cbase,
                                             int lane, int &b, int &hg, int &j, int &ns)
{
    SeqWindow w;
    const int c = chunk_of(cbase, (p.num_seqs + 31) >> 5, g);
    window_load(w, c * 32, cbase[c], p, lane);
    int seqbase, ctx;
    window_find(w, g, true, b, seqbase, ctx, p, cbase, lane);
    const int HG = p.head_groups;
    const int nt = ntiles(ctx);
    const int PT = p.partition_size >> 4;
    const int x = g - seqbase;
    const int nparts = num_parts(ctx, p.partition_size);
    int part = (int)((int64_t)x / ((int64_t)HG * PT));
    if (part > nparts - 1)
        part = nparts - 1;
    const int rem = x - (int)((int64_t)part * HG * PT);
    ns = max(1, min(PT, nt - part * PT));
    hg = rem / ns;
    j = rem - hg * ns;
}

// =====================================================================
// Decode kernel: hpc consumer warps (one per KV head of the group) and one
// producer warp per CTA; launched with 32 * (hpc + 1) threads.
//
// CTA x owns the CTA-tile range [R(x), R(x + 1)).  The stages form a ring;
// each has a "full" mbarrier (the producer arrives with the expected bytes,
// TMA completes them) and an "empty" mbarrier (each consumer warp arrives
// once it is done with the stage).
//
// Mode 0 cuts segments at range borders and merges them inside the kernel.
// Each CTA holding a piece of a cut segment publishes the piece's partial
// state (acc, max, sum, bad) in its slot, then counts itself in at the
// segment's counter with an acquire-release atomic add (segment_arrive).
// The warp whose arrival completes the count merges the segment's head
// after its range (merge_last); everyone else moves on.  No CTA ever waits
// for another: a merge reads only pieces whose arrivals it has counted.
// A stage wait that runs out (bounded, PA_DEV_WAIT_TIMEOUT) makes the warp
// zero the outputs of every segment its range touches, and the CTA counts
// nothing in, so those segments keep zeros.
//
// The kernel is launched as a programmatic dependent of the kernel before it
// on the stream.  Before griddepcontrol.wait it reads only the context
// lengths, the block tables, and the K/V rows of its first tiles that hold
// no sequence's last cached token (the kernel ahead must write none of
// them; the cache write stores only last rows); the query, the last rows,
// the outputs and the workspace come after the wait.  It lets the kernel
// after it start early in the same way.
// =====================================================================
template <typename T, int D, int G, bool MMA, bool TR16, bool KV8>
__global__ void __launch_bounds__(KV8 ? kThreads8 : kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const TileGeo &geo = p.geo;
    const int spw = geo.spw;
    const int hpc = geo.hpc;
    const int total_ctas = gridDim.x;
    const int HG = p.head_groups;
    const int Hq = p.num_q_heads;
    constexpr int SUBS = KV8 ? kSubs8 : 1;   // consumer warps per KV head

    // 1024-byte aligned layout: [stages][full bars][empty bars][meta][score rows][chunk prefix]
    // [merge barriers][exchange areas (FP8)]
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sgen = smem_raw + (sbase - raw);
    const int stages_bytes = spw * geo.stage_bytes;
    const uint32_t full0 = sbase + (uint32_t)stages_bytes;
    const uint32_t empty0 = full0 + 8u * kMaxSpw;
    StageMeta *meta = reinterpret_cast<StageMeta *>(sgen + stages_bytes + 16 * kMaxSpw);
    float *scores_all = reinterpret_cast<float *>(sgen + stages_bytes + 64 * kMaxSpw);
    int *cbase = reinterpret_cast<int *>(scores_all + kMaxHpc * kTile * G);
    // set when a consumer warp of this CTA gave up waiting
    volatile int *cta_lost = cbase + kMaxChunks + 1;
    const uint32_t mbars0 = ptx::smem_u32(sgen + stages_bytes + exchange_off(G));
    uint8_t *xarea = sgen + stages_bytes + exchange_off(G) + kMergeBarBytes;
    constexpr uint32_t kXBars = 32u * 5u * 4u;   // barriers' offset in an exchange area

    if (threadIdx.x == 0) {
        *cta_lost = 0;
        for (int s = 0; s < spw; ++s) {
            ptx::mbar_init(full0 + 8u * s, 1);
            ptx::mbar_init(empty0 + 8u * s, hpc);
        }
        for (int w = 0; w < kMaxHpc * kSubs8; ++w) {
            ptx::mbar_init(mbars0 + 16u * w, 1);
            ptx::mbar_init(mbars0 + 16u * w + 8u, 1);
        }
        if constexpr (SUBS > 1) {
            for (int h = 0; h < hpc; ++h) {
                const uint32_t xb = ptx::smem_u32(xarea + h * exchange_bytes(D)) + kXBars;
                ptx::mbar_init(xb, 1);        // full: the state is in the area
                ptx::mbar_init(xb + 8u, 1);   // free: the state has been read
            }
        }
    }
    ptx::fence_mbar_init();
    // The lengths and block tables are read before the kernel ahead on the
    // stream has completed (see the launch): the work decomposition and the
    // first block-table batches overlap its tail.
    const int total = chunk_prefix(p, cbase);   // contains __syncthreads
    // C <= T CTAs take part, so that every participating range is non-empty
    const int C = min(total_ctas, max(total, 1));
    const int R0 = range_begin(blockIdx.x, C, total, p, cbase, lane);
    const int R1 = range_begin(blockIdx.x + 1, C, total, p, cbase, lane);
    // the next kernel on the stream may start its own set-up on SMs this
    // grid leaves; it waits for this grid to complete before using its results
    if (threadIdx.x == 0)
        ptx::grid_launch_dependents();
    // the producer warp: the last warp of the consumers (bf16, f32), the
    // first of the producer warpgroup (FP8)
    const int pw = KV8 ? kMaxHpc * SUBS : hpc;

    // =================================================== producer warp
    auto producer = [&]() {
        if (R0 >= R1)
            return;
        ptx::prefetch_tensormap(&tmap_k);
        ptx::prefetch_tensormap(&tmap_v);
        const uint64_t policy = ptx::policy_evict_first();
        SeqWindow win;
        {
            const int c = chunk_of(cbase, (p.num_seqs + 31) >> 5, R0);
            window_load(win, c * 32, cbase[c], p, lane);
        }
        TileDesc bat0, bat1;
        fill_batch(bat0, win, R0, R1, p, cbase, lane);
        fill_batch(bat1, win, R0 + 32, R1, p, cbase, lane);
        int filled = 2;
        // Brings the query rows of tile d's segment (this CTA's heads) into
        // L2; no value is read.
        auto prefetch_query = [&](const TileDesc &d) {
            const uint8_t *qsrc = static_cast<const uint8_t *>(p.q) +
                                  ((int64_t)d.b * Hq + (int64_t)d.h * hpc * G) * D * sizeof(T);
            for (int off = lane * 128; off < hpc * geo.q_head_bytes; off += 32 * 128)
                ptx::prefetch_l2(qsrc + off);
        };
        // Fills ring position k with tile R0 + k (descriptor d): the
        // metadata, the expected bytes, and the K/V copies (kv) and/or the
        // segment's query rows (q).  False if the bounded wait for the stage
        // ran out.
        auto issue = [&](int k, const TileDesc &d, bool kv, bool q) -> bool {
            const int s = k % spw;
            const uint32_t bar = full0 + 8u * s;
            if (kv && k >= spw &&
                !ptx::mbar_wait_bounded(empty0 + 8u * s, (uint32_t)(((k / spw) - 1) & 1),
                                        p.wait_ns)) {
                if (lane == 0)
                    report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                return false;
            }
            // the first tile of each consumer warp of a head in the segment
            // carries the segment's query rows
            const bool newseg = d.j < SUBS || k < SUBS;
            const uint32_t stage = sbase + (uint32_t)(s * geo.stage_bytes);
            // test hook: the copies of this CTA's second tile are not issued,
            // so the stage never completes and the bounded waits run out
            const bool withhold = (int)blockIdx.x == p.withhold_cta && k == 1;
            const int h0 = d.h * hpc;
            // (the first tile's query rows are read by the consumer warps
            // themselves, straight after their wait)
            const bool qcopy = newseg && k != 0;
            if (kv && lane == 0) {
                int tx = qcopy ? geo.q_bytes : 0;
                bool bad = false;
#pragma unroll
                for (int bx = 0; bx < 4; ++bx) {
                    if (bx < geo.bpt && bx * geo.tr < d.n) {
                        if (d.phys[bx] < 0 || (int64_t)d.phys[bx] >= p.num_blocks)
                            bad = true;
                        else
                            tx += 2 * geo.box_tx;
                    }
                }
                StageMeta m;
                m.b = d.b;
                m.hg = d.h;
                m.part = d.part;
                m.j = d.j;
                m.ns = d.ns;
                m.n = d.n;
                m.ctx = d.ctx;
                m.bad = bad ? 1 : 0;
                m.k = k;
                m.nt = 1;
                m.n1 = 0;
                m.end = 0;
                meta[s] = m;
                // release: consumers see the metadata once the phase completes
                ptx::mbar_arrive_expect_tx(bar, (uint32_t)tx);
#pragma unroll
                for (int bx = 0; bx < 4; ++bx) {
                    if (bx >= geo.bpt || bx * geo.tr >= d.n || d.phys[bx] < 0 ||
                        (int64_t)d.phys[bx] >= p.num_blocks || withhold)
                        continue;
                    const int row =
                        d.phys[bx] * p.block_size + ((d.t0 + bx * geo.tr) & (p.block_size - 1));
                    const uint32_t off = (uint32_t)(bx * geo.box_stride);
                    ptx::tma_load_4d(stage + off, &tmap_k, 0, row, 0, h0, bar, policy);
                    ptx::tma_load_4d(stage + (uint32_t)geo.kv_bytes + off, &tmap_v, 0, row, 0, h0,
                                     bar, policy);
                }
            }
            if (q && qcopy && !withhold && lane == 0 && geo.q_bytes > 0) {
                const T *qsrc = static_cast<const T *>(p.q) + ((int64_t)d.b * Hq + (int64_t)h0 * G) * D;
                ptx::bulk_g2s(stage + (uint32_t)geo.q_off, qsrc, (uint32_t)geo.q_bytes, bar);
            }
            if constexpr (KV8) {
                // FP8 stages carry no query rows: the consumers read them
                // from global memory when they start the segment; bring
                // them into L2 now
                if (q && (d.j == 0 || k == 0))
                    prefetch_query(d);
            }
            __syncwarp();
            return true;
        };
        // Before the kernel ahead has completed, the K/V rows of the range's
        // first tiles are already fetched, as long as none of them holds its
        // sequence's last cached token: that row is the only one the cache
        // write ahead of this kernel stores.  Their query rows come after the
        // wait, as everything else.
        // Their segments' query rows are prefetched into L2 meanwhile (no
        // value is read before the wait; L2 keeps the latest writes).
        int early = 0;
        for (; early < min(spw, R1 - R0); ++early) {
            const TileDesc d = shfl_desc(bat0, early);
            if (d.t0 + d.n >= d.ctx)
                break;
            issue(early, d, true, false);
            if (d.j == 0 || early == 0)
                prefetch_query(d);
        }
        // the query, the last rows and the outputs may be written or read by
        // the kernel ahead
        ptx::grid_wait_prerequisites();
        for (int k = 0; k < early; ++k)
            issue(k, shfl_desc(bat0, k), false, true);
        int issued = R0 + early;
        for (; issued < R1; ++issued) {
            const int i = issued;
            const int k = i - R0;
            const TileDesc d = ((k >> 5) & 1) ? shfl_desc(bat1, k & 31) : shfl_desc(bat0, k & 31);
            if (!issue(k, d, true, true))
                break;
            // descriptors of batch k/32 are used up: prepare the batch after next
            if ((k & 31) == 31) {
                if (filled & 1)
                    fill_batch(bat1, win, R0 + 32 * filled, R1, p, cbase, lane);
                else
                    fill_batch(bat0, win, R0 + 32 * filled, R1, p, cbase, lane);
                ++filled;
            }
        }
        if (issued < R1) {
            // aborted: let copies still in flight land before exiting (bounded)
            for (int i = max(R0, issued - spw); i < issued; ++i) {
                const int k = i - R0;
                ptx::mbar_wait_bounded(full0 + 8u * (k % spw), (uint32_t)((k / spw) & 1),
                                       p.wait_ns);
            }
        }
    };
    // ============================================ producer warp (FP8 cache)
    // A stage holds two consecutive tiles of one segment when the range has
    // them (tile k pairs with k + 1 if both lie in the same segment inside
    // the range), else one; the consumer warps of a head take alternate
    // stages.  After the last stage come SUBS end stages (no tiles), one per
    // consumer warp of a head.
    auto producer8 = [&]() {
        if (R0 >= R1)
            return;
        ptx::prefetch_tensormap(&tmap_k);
        ptx::prefetch_tensormap(&tmap_v);
        const uint64_t policy = ptx::policy_evict_first();
        SeqWindow win;
        {
            const int c = chunk_of(cbase, (p.num_seqs + 31) >> 5, R0);
            window_load(win, c * 32, cbase[c], p, lane);
        }
        TileDesc bat0, bat1;
        fill_batch(bat0, win, R0, R1, p, cbase, lane);
        fill_batch(bat1, win, R0 + 32, R1, p, cbase, lane);
        int loaded = 1;   // batches 0 and 1 are in bat0, bat1
        // descriptor of tile R0 + k (whole warp; k only grows, by 1 or 2)
        auto desc = [&](int k) -> TileDesc {
            const int bt = k >> 5;
            if (bt > loaded) {
                // batch bt replaces batch bt - 2, whose tiles are all issued
                if (bt & 1)
                    fill_batch(bat1, win, R0 + 32 * bt, R1, p, cbase, lane);
                else
                    fill_batch(bat0, win, R0 + 32 * bt, R1, p, cbase, lane);
                loaded = bt;
            }
            return (bt & 1) ? shfl_desc(bat1, k & 31) : shfl_desc(bat0, k & 31);
        };
        auto prefetch_query = [&](const TileDesc &d) {
            const uint8_t *qsrc = static_cast<const uint8_t *>(p.q) +
                                  ((int64_t)d.b * Hq + (int64_t)d.h * hpc * G) * D * sizeof(T);
            for (int off = lane * 128; off < hpc * geo.q_head_bytes; off += 32 * 128)
                ptx::prefetch_l2(qsrc + off);
        };
        auto tile_ok = [&](const TileDesc &d, int bx) {
            return d.phys[bx] >= 0 && (int64_t)d.phys[bx] < p.num_blocks;
        };
        // Fills stage q with tiles R0 + k (d0) and, when `pair`, R0 + k + 1
        // (d1).  False if the bounded wait for the stage ran out.
        auto issue = [&](int q, int k, const TileDesc &d0, bool pair,
                         const TileDesc &d1) -> bool {
            const int s = q % spw;
            const uint32_t bar = full0 + 8u * s;
            if (q >= spw &&
                !ptx::mbar_wait_bounded(empty0 + 8u * s, (uint32_t)(((q / spw) - 1) & 1),
                                        p.wait_ns)) {
                if (lane == 0)
                    report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                return false;
            }
            const uint32_t stage = sbase + (uint32_t)(s * geo.stage_bytes);
            // test hook: the copies of this CTA's second stage are not issued,
            // so the stage never completes and the bounded waits run out
            const bool withhold = (int)blockIdx.x == p.withhold_cta && q == 1;
            const int h0 = d0.h * hpc;
            if (lane == 0) {
                int tx = 0;
                bool bad = false;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const TileDesc &d = t ? d1 : d0;
                    if (t == 1 && !pair)
                        continue;
#pragma unroll
                    for (int bx = 0; bx < 4; ++bx) {
                        if (bx < geo.bpt && bx * geo.tr < d.n) {
                            if (!tile_ok(d, bx))
                                bad = true;
                            else
                                tx += 2 * geo.box_tx;
                        }
                    }
                }
                StageMeta m;
                m.b = d0.b;
                m.hg = d0.h;
                m.part = d0.part;
                m.j = d0.j;
                m.ns = d0.ns;
                m.n = d0.n;
                m.ctx = d0.ctx;
                m.bad = bad ? 1 : 0;
                m.k = k;
                m.nt = pair ? 2 : 1;
                m.n1 = pair ? d1.n : 0;
                m.end = 0;
                meta[s] = m;
                // release: consumers see the metadata once the phase completes
                ptx::mbar_arrive_expect_tx(bar, (uint32_t)tx);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const TileDesc &d = t ? d1 : d0;
                    if ((t == 1 && !pair) || withhold)
                        continue;
#pragma unroll
                    for (int bx = 0; bx < 4; ++bx) {
                        if (bx >= geo.bpt || bx * geo.tr >= d.n || !tile_ok(d, bx))
                            continue;
                        const int row = d.phys[bx] * p.block_size +
                                        ((d.t0 + bx * geo.tr) & (p.block_size - 1));
                        const uint32_t off = (uint32_t)(t * geo.kv_bytes + bx * geo.box_stride);
                        ptx::tma_load_4d(stage + off, &tmap_k, 0, row, 0, h0, bar, policy);
                        ptx::tma_load_4d(stage + (uint32_t)(2 * geo.kv_bytes) + off, &tmap_v, 0,
                                         row, 0, h0, bar, policy);
                    }
                }
            }
            __syncwarp();
            return true;
        };
        const int nk = R1 - R0;
        int k = 0, q = 0;
        TileDesc d0, d1;
        bool pair = false;
        auto next = [&]() {
            d0 = desc(k);
            pair = k + 1 < nk && d0.j + 1 < d0.ns;
            d1 = pair ? desc(k + 1) : d0;
        };
        // Before the kernel ahead has completed, the K/V rows of the first
        // stages are already fetched, as long as none of their tiles holds its
        // sequence's last cached token (the only row the cache write ahead of
        // this kernel stores), and their segments' query rows are prefetched
        // into L2 (no value is read before the wait).
        for (; q < spw && k < nk; ++q) {
            next();
            if (d0.t0 + d0.n >= d0.ctx || (pair && d1.t0 + d1.n >= d1.ctx))
                break;
            issue(q, k, d0, pair, d1);
            if (d0.j == 0 || k == 0)
                prefetch_query(d0);
            k += pair ? 2 : 1;
        }
        ptx::grid_wait_prerequisites();
        bool ok = true;
        for (; k < nk; ++q) {
            next();
            if (!(ok = issue(q, k, d0, pair, d1)))
                break;
            if (d0.j == 0 || k == 0)
                prefetch_query(d0);
            k += pair ? 2 : 1;
        }
        // one end stage per consumer warp of a head (no copies: the arrival
        // completes the phase)
        for (int t = 0; ok && t < SUBS; ++t, ++q) {
            const int s = q % spw;
            if (q >= spw &&
                !ptx::mbar_wait_bounded(empty0 + 8u * s, (uint32_t)(((q / spw) - 1) & 1),
                                        p.wait_ns)) {
                if (lane == 0)
                    report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                ok = false;
                break;
            }
            if (lane == 0) {
                StageMeta m = {};
                m.end = 1;
                meta[s] = m;
                ptx::mbar_arrive(full0 + 8u * s);
            }
            __syncwarp();
        }
        if (!ok) {
            // aborted: let copies still in flight land before exiting (bounded)
            for (int x = max(0, q - spw); x < q; ++x)
                ptx::mbar_wait_bounded(full0 + 8u * (x % spw), (uint32_t)((x / spw) & 1),
                                       p.wait_ns);
        }
    };
    if constexpr (KV8) {
        // each role's code runs under its own register count
        if (warp >= kMaxHpc * SUBS) {
            ptx::setmaxnreg_dec<kRegsProducer8>();
            if (warp == pw)
                producer8();
            return;
        }
        ptx::setmaxnreg_inc<kRegsConsumer8>();
        if (warp >= hpc * SUBS)
            return;   // no work for this warp
    } else if (warp == pw) {
        producer();
        return;
    }

    // ====================================================== consumer warps
    const int hl = warp % hpc;                  // head within the group
    const int sub = warp / hpc;                 // which of the head's SUBS warps
    const int hline = hl * geo.head_lines;      // its first 128-byte line in a box
    float *scores = scores_all + hl * kTile * G;
    // outputs and the workspace may still be in use by the kernel ahead
    ptx::grid_wait_prerequisites();

    // Sequences without tiles (length 0 or invalid) get a zero output.
    for (int b = blockIdx.x; sub == 0 && b < p.num_seqs; b += total_ctas) {
        const int rawc = p.context_lens[b];
        if (eff_ctx(rawc, p.ctx_cap) > 0)
            continue;
        if (rawc != 0 && lane == 0 && hl == 0)
            report(p.dev_status, PA_DEV_BAD_CONTEXT);
        for (int hg = 0; hg < HG; ++hg) {
            const int64_t bh0 = (int64_t)b * Hq + (int64_t)(hg * hpc + hl) * G;
            T *o = static_cast<T *>(p.out) + bh0 * D;
            for (int i = lane; i < G * D; i += 32)
                store_out<T>(o + i, 0.f);
            if (p.public_partials) {
                for (int g = 0; g < G; ++g) {
                    const int64_t slot = (bh0 + g) * p.max_parts;
                    for (int e = lane; e < D; e += 32)
                        p.tmp_out[slot * D + e] = 0.f;
                    if (lane == 0) {
                        p.max_logits[slot] = -INFINITY;
                        p.exp_sums[slot] = 0.f;
                    }
                }
            }
        }
    }

    static_assert(!KV8 || (MMA && TR16), "an FP8 cache uses the tensor-core math, blocks >= 16");
    using Math = typename std::conditional<
        KV8, MmaMath8<D, G>,
        typename std::conditional<MMA, MmaMath<D, G, TR16>, SimtMath<T, D, G, TR16>>::type>::type;
    Math math;
    int segS = 0;          // global index of the current segment's first tile
    bool seg_bad = false;
    bool timed_out = false;
    int lost = R1;         // first tile of the range lost to a wait that ran out
    int xc = 0;            // state exchanges so far between the head's two warps (FP8)
    // cut segments this warp merges (mode 0): one met at the start of the
    // range, one that runs past its end
    // (its first CTA and piece count, sequence and head group)
    int laterS = -1, laterX = 0, laterN = 0, laterB = 0, laterHG = 0;
    int firstS = -1, firstX = 0, firstN = 0, firstB = 0, firstHG = 0;

    // this CTA's arrival counters start the call at (epoch, 0) unless an
    // arrival has already counted in them (see segment_arrive)
    if (p.mode == 0 && lane == 0 && sub == 0)
        ptx::red_max_relaxed_gpu_u64(counter_of(p, blockIdx.x, hl),
                                     (unsigned long long)p.epoch << 32);

    // Stage q of the ring holds tile R0 + q (bf16, f32) or one or two
    // consecutive tiles of one segment (FP8 cache, see producer8); with SUBS
    // warps per head, warp `sub` takes stages sub, sub + SUBS, ...
    int done = R0;        // tiles of the range up to this warp's last stage
    int seg_prev = -1;    // segment of this warp's last stage
    for (int q = sub;; q += SUBS) {
        // (an FP8 producer marks the end of a non-empty range with end stages)
        if (KV8 ? R0 >= R1 : R0 + q >= R1)
            break;
        const int s = q % spw;
        if (!ptx::mbar_wait_bounded(full0 + 8u * s, (uint32_t)((q / spw) & 1), p.wait_ns)) {
            if (lane == 0)
                report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
            timed_out = true;
            lost = done;
            break;
        }
        const StageMeta d = meta[s];
        if constexpr (KV8) {
            if (d.end)
                break;
        }
        // the stage's first and last tiles
        const int nt = KV8 ? d.nt : 1;
        const int i = KV8 ? R0 + d.k : R0 + q;
        const int i_end = i + nt - 1;
        const bool newseg = i - d.j != seg_prev;   // this warp's first stage of the segment
        const uint32_t kreg = sbase + (uint32_t)(s * geo.stage_bytes);
        const uint32_t vreg = kreg + (uint32_t)(geo.tps * geo.kv_bytes);
        const uint8_t *qslot = sgen + s * geo.stage_bytes + geo.q_off + hl * geo.q_head_bytes;
        if (newseg) {
            segS = i - d.j;
            seg_prev = segS;
            seg_bad = false;
            if constexpr (KV8)
                math.begin(static_cast<const uint8_t *>(p.q) +
                               ((int64_t)d.b * Hq + (int64_t)(d.hg * hpc + hl) * G) * D * 2,
                           lane, p.scale_log2);
            else {
                if (q == 0) {
                    // the range's first stage carries no query rows: this
                    // warp copies its head's rows into the slot
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        static_cast<const T *>(p.q) +
                        ((int64_t)d.b * Hq + (int64_t)(d.hg * hpc + hl) * G) * D);
                    uint4 *dst = reinterpret_cast<uint4 *>(const_cast<uint8_t *>(qslot));
                    for (int u = lane; u < geo.q_head_bytes / 16; u += 32)
                        dst[u] = __ldg(src + u);
                    __syncwarp();
                }
                if constexpr (MMA)
                    math.begin(qslot, lane);
                else
                    math.begin(qslot, lane, p.scale_log2);
            }
        }
        if (d.bad)
            seg_bad = true;
        if (!seg_bad) {
            // V rows past the sequence end hold whatever the pool has there:
            // zero them in this head's V (their weight is 0, but 0 * NaN is NaN)
#pragma unroll 1
            for (int t = 0; t < nt; ++t) {
                const int n = t ? d.n1 : d.n;
                const uint32_t vt = vreg + (uint32_t)(t * geo.kv_bytes);
                if (n < kTile) {
                    constexpr int NCH = D * (KV8 ? 1 : (int)sizeof(T)) / 128;
                    const int lines = (kTile - n) * NCH;
                    for (int idx = lane; idx < lines * 8; idx += 32) {
                        const int line = idx >> 3;
                        const int tk = n + line / NCH;
                        const int ch = line % NCH;
                        const uint32_t a = tile_addr<TR16>(vt, hline, tk, ch * 8 + (idx & 7), geo);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0)
                                     : "memory");
                    }
                    __syncwarp();
                }
            }
#pragma unroll 1
            for (int t = 0; t < nt; ++t) {
                const int n = t ? d.n1 : d.n;
                const uint32_t kt = kreg + (uint32_t)(t * geo.kv_bytes);
                const uint32_t vt = vreg + (uint32_t)(t * geo.kv_bytes);
                if constexpr (MMA)
                    math.tile(kt, vt, hline, n, p.scale_log2, geo, lane);
                else
                    math.tile(kt, vt, hline, n, scores, geo, lane);
            }
        }
        done = i_end + 1;
        const int last = min(segS + d.ns, R1) - 1;   // the segment's last tile in the range
        const bool is_final = i_end == last;
        // (FP8) the warp whose stage comes just before the segment's final one
        // (the other warp's) hands its partial state over and keeps its stage:
        // the state goes through the stage's lines of its head.  The final
        // stage holds the segment's last one or two tiles.
        const bool hand_over = SUBS > 1 && !is_final && last - i_end <= 2;
        if (!hand_over) {
            // the stage may be refilled: order this warp's shared-memory
            // accesses before the producer's next TMA into it, then release it
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(empty0 + 8u * s);
        }

        // ---- end of this warp's share of a segment (or of this CTA's range)
        if (is_final || hand_over) {
            if constexpr (SUBS > 1) {
                // Two warps per head: the one holding the segment's last tile
                // in the range completes it; the other hands it its partial
                // state (bounded waits).
                float *st = reinterpret_cast<float *>(xarea + hl * exchange_bytes(D));
                const uint32_t xfull = ptx::smem_u32(st) + kXBars, xfree = xfull + 8u;
                auto head_lines = [&](int stage, int v) {
                    return reinterpret_cast<float *>(sgen + stage * geo.stage_bytes +
                                                     v * geo.tps * geo.kv_bytes + hline * 128);
                };
                if (hand_over) {
                    if (xc > 0 &&
                        !ptx::mbar_wait_bounded(xfree, (uint32_t)((xc - 1) & 1), p.wait_ns)) {
                        if (lane == 0)
                            report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                        timed_out = true;
                        lost = i;
                        break;
                    }
                    __syncwarp();
                    math.save(head_lines(s, 0), head_lines(s, 1), st, seg_bad, lane);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0)
                        ptx::mbar_arrive(xfull);
                    ++xc;
                    continue;
                }
                if (max(segS, R0) < i) {
                    if (!ptx::mbar_wait_bounded(xfull, (uint32_t)(xc & 1), p.wait_ns)) {
                        if (lane == 0)
                            report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                        timed_out = true;
                        lost = i;
                        break;
                    }
                    // the other warp's last stage of the segment is q - 1
                    const int sh = (q - 1) % spw;
                    seg_bad |= math.absorb(head_lines(sh, 0), head_lines(sh, 1), st, lane);
                    // its stage may be refilled now (released on its behalf)
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        ptx::mbar_arrive(empty0 + 8u * sh);
                        ptx::mbar_arrive(xfree);
                    }
                    ++xc;
                }
            }
            math.finish();
            const int segE = segS + d.ns;
            const bool complete = segS >= R0 && segE <= R1;
            const int64_t bh0 = (int64_t)d.b * Hq + (int64_t)(d.hg * hpc + hl) * G;
            if (p.mode == 0 && !complete) {
                // a piece of a cut segment: publish it, merge after the range
                const bool first = segS >= R0;
                const int slot = piece_slot(blockIdx.x, first, hpc, hl);
                float *ps = p.wpart + (int64_t)slot * p.slot_floats;
                // the accumulator in the output's type (bf16 rounds it once)
                constexpr int SOT = piece_stats_off(D, G, (int)sizeof(T));
                math.template publish<T>(ps, lane);
                math.publish_stats(ps + SOT, lane);
                if (lane == 0)
                    ps[SOT + 2 * G] = seg_bad ? 1.f : 0.f;
                // the warp barrier orders every lane's stores before lane 0's
                // release (the counter update)
                __syncwarp();
                const int x0 = cta_of(segS, C, total);
                const int np = cta_of(segS + d.ns - 1, C, total) - x0 + 1;
                int arrived = 0;
                if (lane == 0)
                    arrived = segment_arrive(counter_of(p, x0, hl), p.epoch);
                arrived = __shfl_sync(kFull, arrived, 0);
                __syncwarp();
                if (arrived == 0) {
                    if (lane == 0)
                        report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                    continue;
                }
                if (arrived != np)
                    continue;   // a later arrival merges the segment
                if (first) {
                    firstS = segS;
                    firstX = x0;
                    firstN = np;
                    firstB = d.b;
                    firstHG = d.hg;
                } else {
                    laterS = segS;
                    laterX = x0;
                    laterN = np;
                    laterB = d.b;
                    laterHG = d.hg;
                }
                continue;
            }
            if (seg_bad && lane == 0)
                report(p.dev_status, PA_DEV_BAD_BLOCK);
            const bool single = num_parts(d.ctx, p.partition_size) == 1;
            if (single && !p.public_partials) {
                if constexpr (KV8)
                    math.store_final(static_cast<T *>(p.out) + bh0 * D, seg_bad, p.out_scale, lane);
                else
                    math.store_final(static_cast<T *>(p.out) + bh0 * D, seg_bad, lane);
                continue;
            }
            math.for_each(
                lane,
                [&](int hh, int e, float v, float ll) {
                    const float res = (seg_bad || !(ll > 0.f)) ? 0.f : v / ll;
                    if (p.public_partials)
                        p.tmp_out[((bh0 + hh) * p.max_parts + d.part) * D + e] = res;
                    if (single)
                        store_out<T>(static_cast<T *>(p.out) + (bh0 + hh) * D + e,
                                     res * p.out_scale);
                },
                [&](int hh, float mm, float ll) {
                    if (p.public_partials) {
                        const int64_t slot = (bh0 + hh) * p.max_parts + d.part;
                        const bool empty = seg_bad || !(ll > 0.f);
                        p.max_logits[slot] = empty ? -INFINITY : mm / kLog2e;
                        p.exp_sums[slot] = empty ? 0.f : ll;
                    }
                });
        }
    }

    auto zero_segment = [&](int b, int hg) {
        T *o = static_cast<T *>(p.out) + ((int64_t)b * Hq + (int64_t)(hg * hpc + hl) * G) * D;
        for (int e = lane; e < G * D; e += 32)
            store_out<T>(o + e, 0.f);
    };
    if (timed_out) {
        // the rest of the range is lost: zero this warp's head of every
        // segment from the lost tile on (their pieces here are never counted
        // in, so no merge overwrites the zeros), and of the segments this
        // warp was to merge; the CTA's other warps do the same for their heads
        for (int g = lost; g < R1;) {
            int b, hg, j, ns;
            tile_segment(g, p, cbase, lane, b, hg, j, ns);
            zero_segment(b, hg);
            g += ns - j;
        }
        if (laterS >= 0)
            zero_segment(laterB, laterHG);
        if (firstS >= 0)
            zero_segment(firstB, firstHG);
        if (lane == 0)
            *cta_lost = 1;
    }
    if (p.mode == 0) {
        // every consumer warp is past its last stage (and with it every copy
        // into the ring has landed): the ring is free scratch for the merges
        asm volatile("bar.sync 1, %0;" ::"r"(32 * hpc * SUBS) : "memory");
        if (timed_out)
            return;
        if (*cta_lost != 0) {
            // another warp of this CTA gave up: copies into the ring may still
            // be landing, so it is no scratch; the segments this warp was to
            // merge get zeros, as lost ones
            if (laterS >= 0 || firstS >= 0) {
                if (lane == 0)
                    report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                if (laterS >= 0)
                    zero_segment(laterB, laterHG);
                if (firstS >= 0)
                    zero_segment(firstB, firstHG);
            }
            return;
        }
        const int cap = (int)((int64_t)stages_bytes / (hpc * SUBS) & ~(int64_t)127);
        uint8_t *buf = sgen + (int64_t)warp * cap;
        uint32_t mphase = 0;
        auto merge = [&](int x0, int np, int B0, int HG0) {
            merge_last<T, D, G, Math>(p, x0, np,
                                      (int64_t)B0 * Hq + (int64_t)(HG0 * hpc + hl) * G, hl, buf,
                                      cap, mbars0 + 16u * (uint32_t)warp, mphase, lane);
        };
        if (laterS >= 0)
            merge(laterX, laterN, laterB, laterHG);
        if (firstS >= 0)
            merge(firstX, firstN, firstB, firstHG);
    }
}

// =====================================================================
// Explicit split-K reduce: one CTA per (sequence, query head).
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
