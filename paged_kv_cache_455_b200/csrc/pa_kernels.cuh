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
//     mode 0 (stream-K): equal ranges.  A segment cut by range boundaries
//       leaves one partial softmax state per piece and head (at most two
//       pieces per CTA), merged afterwards by merge_kernel.  Balanced for any
//       mix of lengths.
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
// merge_kernel    log-sum-exp merge of the warp pieces of cut segments.
// reduce_kernel   log-sum-exp merge of fixed-size partitions (explicit API).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <type_traits>

#include "pa.h"
#include "pa_ptx.cuh"

namespace pa {

#ifndef PA_MAX_SPW
#define PA_MAX_SPW 4
#endif

constexpr int kMaxHpc = 4;                  // KV heads per CTA tile, at most
constexpr int kThreads = 32 * (kMaxHpc + 1);// launch bound: consumers + producer
constexpr int kMaxSpw = PA_MAX_SPW;         // stages in the ring, at most
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
    int kv_bytes;      // bytes of a K (or V) region
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
    int32_t *seg_start;      // mode 0: first global tile of each (b, head group) segment
    int32_t *total_tiles;    // mode 0: total tile count (written by the kernel)
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
    float scale_log2;
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

struct MergeParams {
    void *out;
    const float *wpart;
    const int32_t *seg_start;
    const int32_t *total_tiles;
    const int32_t *context_lens;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int ctx_cap;
    int total_ctas;
    int hpc;
    int slot_floats;
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

// =====================================================================
// Tile enumeration
// =====================================================================
__device__ __forceinline__ int eff_ctx(int ctx, int cap) { return (ctx < 0 || ctx > cap) ? 0 : ctx; }
__device__ __forceinline__ int num_parts(int ctx, int P) { return ctx <= 0 ? 1 : (ctx + P - 1) / P; }
__device__ __forceinline__ int ntiles(int ctx) { return (ctx + kTile - 1) / kTile; }

// Total tiles of the batch (every lane gets it).
__device__ __forceinline__ int count_tiles(const DecodeParams &p, int lane)
{
    int sum = 0;
    for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
        const int b = b0 + lane;
        if (b < p.num_seqs)
            sum += ntiles(eff_ctx(p.context_lens[b], p.ctx_cap)) * p.head_groups;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        sum += __shfl_xor_sync(kFull, sum, o);
    return sum;
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

// Resolves each lane's global tile index g (ignored where !want) to its
// sequence: b, the global index of the sequence's first tile, and its
// effective length.  The window only moves forward, so targets must not
// precede it.  Warp-uniform control flow.
__device__ __forceinline__ void window_find(SeqWindow &w, int g, bool want, int &b, int &seqbase,
                                            int &ctx, const DecodeParams &p, int lane)
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
        window_load(w, w.b0 + 32, last, p, lane);
    }
}

// Tile descriptor (h is the head group); a batch holds 32 consecutive tiles,
// one per lane.
struct TileDesc {
    int b, h, part, j, ns, t0, n, ctx;
    int phys[4];
};

// Descriptor of lane `src` of batch d1 (sel) or d0 (!sel), to every lane.
__device__ __forceinline__ TileDesc shfl_desc(const TileDesc &d0, const TileDesc &d1, bool sel,
                                              int src)
{
    TileDesc o;
    o.b = __shfl_sync(kFull, sel ? d1.b : d0.b, src);
    o.h = __shfl_sync(kFull, sel ? d1.h : d0.h, src);
    o.part = __shfl_sync(kFull, sel ? d1.part : d0.part, src);
    o.j = __shfl_sync(kFull, sel ? d1.j : d0.j, src);
    o.ns = __shfl_sync(kFull, sel ? d1.ns : d0.ns, src);
    o.t0 = __shfl_sync(kFull, sel ? d1.t0 : d0.t0, src);
    o.n = __shfl_sync(kFull, sel ? d1.n : d0.n, src);
    o.ctx = __shfl_sync(kFull, sel ? d1.ctx : d0.ctx, src);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        o.phys[k] = __shfl_sync(kFull, sel ? d1.phys[k] : d0.phys[k], src);
    return o;
}

// Fills the descriptors of tiles [base, base + 32) below `end` and starts
// their block-table loads.
__device__ __forceinline__ void fill_batch(TileDesc &d, SeqWindow &w, int base, int end,
                                           const DecodeParams &p, int lane)
{
    const int g = base + lane;
    const bool want = g < end;
    int b, seqbase, ctx;
    window_find(w, g, want, b, seqbase, ctx, p, lane);
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
                                           int lane)
{
    if (gw >= total_warps)
        return T;
    const int x = (int)((int64_t)gw * T / total_warps);
    if (p.mode == 0 || x >= T)
        return x;
    // mode 1: the first segment start at or after x
    SeqWindow w;
    window_load(w, 0, 0, p, lane);
    TileDesc d;
    fill_batch(d, w, x, x + 1, p, lane);
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

// Bytes of the decode kernel's dynamic shared memory besides the stages:
// alignment slack, full and empty barriers, per-stage tile metadata, and the
// CUDA-core math's score rows.
__host__ __device__ constexpr int decode_smem_fixed(int G)
{
    return 1024 + 16 * kMaxSpw + 32 * kMaxSpw + kMaxHpc * kTile * G * 4;
}

// Tile metadata the producer warp hands to the consumer warps with a stage.
struct StageMeta {
    int b, hg, part, j, ns, n, ctx, bad;
};

// =====================================================================
// Decode kernel: hpc consumer warps (one per KV head of the group) and one
// producer warp per CTA; launched with 32 * (hpc + 1) threads.
//
// CTA x owns the CTA-tile range [range_begin(x), range_begin(x + 1)).  The
// stages form a ring; each has a "full" mbarrier (the producer arrives with
// the expected bytes, TMA completes them) and an "empty" mbarrier (each
// consumer warp arrives once it is done with the stage).  No warp waits on
// another CTA, and every wait is bounded.
// =====================================================================
template <typename T, int D, int G, bool MMA, bool TR16>
__global__ void __launch_bounds__(kThreads, 1)
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

    // 1024-byte aligned layout: [stages][full bars][empty bars][meta][score rows]
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sgen = smem_raw + (sbase - raw);
    const int stages_bytes = spw * geo.stage_bytes;
    const uint32_t full0 = sbase + (uint32_t)stages_bytes;
    const uint32_t empty0 = full0 + 8u * kMaxSpw;
    StageMeta *meta = reinterpret_cast<StageMeta *>(sgen + stages_bytes + 16 * kMaxSpw);
    float *scores_all = reinterpret_cast<float *>(sgen + stages_bytes + 48 * kMaxSpw);

    if (threadIdx.x == 0) {
        for (int s = 0; s < spw; ++s) {
            ptx::mbar_init(full0 + 8u * s, 1);
            ptx::mbar_init(empty0 + 8u * s, hpc);
        }
    }
    ptx::fence_mbar_init();
    __syncthreads();

    const int total = count_tiles(p, lane);
    const int R0 = range_begin(blockIdx.x, total_ctas, total, p, lane);
    const int R1 = range_begin(blockIdx.x + 1, total_ctas, total, p, lane);

    if (warp == hpc) {
        // =================================================== producer warp
        if (R0 >= R1)
            return;
        ptx::prefetch_tensormap(&tmap_k);
        ptx::prefetch_tensormap(&tmap_v);
        const uint64_t policy = ptx::policy_evict_first();
        SeqWindow win;
        window_load(win, 0, 0, p, lane);
        TileDesc bat0, bat1;
        fill_batch(bat0, win, R0, R1, p, lane);
        fill_batch(bat1, win, R0 + 32, R1, p, lane);
        int filled = 2;
        int issued = R0;
        for (; issued < R1; ++issued) {
            const int i = issued;
            const int k = i - R0;
            const int s = k % spw;
            const uint32_t bar = full0 + 8u * s;
            if (k >= spw && !ptx::mbar_wait_bounded(empty0 + 8u * s,
                                                    (uint32_t)(((k / spw) - 1) & 1), kWaitLimitNs)) {
                if (lane == 0)
                    report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                break;
            }
            const TileDesc d = shfl_desc(bat0, bat1, (k >> 5) & 1, k & 31);
            const bool newseg = d.j == 0 || i == R0;
            int tx = newseg ? geo.q_bytes : 0;
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
            const uint32_t stage = sbase + (uint32_t)(s * geo.stage_bytes);
            if (lane == 0) {
                StageMeta m;
                m.b = d.b;
                m.hg = d.h;
                m.part = d.part;
                m.j = d.j;
                m.ns = d.ns;
                m.n = d.n;
                m.ctx = d.ctx;
                m.bad = bad ? 1 : 0;
                meta[s] = m;
                // release: consumers see the metadata once the phase completes
                ptx::mbar_arrive_expect_tx(bar, (uint32_t)tx);
                const int h0 = d.h * hpc;
#pragma unroll
                for (int bx = 0; bx < 4; ++bx) {
                    if (bx >= geo.bpt || bx * geo.tr >= d.n || d.phys[bx] < 0 ||
                        (int64_t)d.phys[bx] >= p.num_blocks)
                        continue;
                    const int row =
                        d.phys[bx] * p.block_size + ((d.t0 + bx * geo.tr) & (p.block_size - 1));
                    const uint32_t off = (uint32_t)(bx * geo.box_stride);
                    ptx::tma_load_4d(stage + off, &tmap_k, 0, row, 0, h0, bar, policy);
                    ptx::tma_load_4d(stage + (uint32_t)geo.kv_bytes + off, &tmap_v, 0, row, 0, h0,
                                     bar, policy);
                }
                if (newseg) {
                    const T *qsrc =
                        static_cast<const T *>(p.q) + ((int64_t)d.b * Hq + (int64_t)h0 * G) * D;
                    ptx::bulk_g2s(stage + (uint32_t)geo.q_off, qsrc, (uint32_t)geo.q_bytes, bar);
                }
            }
            __syncwarp();
            // descriptors of batch k/32 are used up: prepare the batch after next
            if ((k & 31) == 31) {
                if (filled & 1)
                    fill_batch(bat1, win, R0 + 32 * filled, R1, p, lane);
                else
                    fill_batch(bat0, win, R0 + 32 * filled, R1, p, lane);
                ++filled;
            }
        }
        if (issued < R1) {
            // aborted: let copies still in flight land before exiting (bounded)
            for (int i = max(R0, issued - spw); i < issued; ++i) {
                const int k = i - R0;
                ptx::mbar_wait_bounded(full0 + 8u * (k % spw), (uint32_t)((k / spw) & 1),
                                       kWaitLimitNs);
            }
        }
        return;
    }

    // ====================================================== consumer warps
    const int hl = warp;                        // head within the group
    const int hline = hl * geo.head_lines;      // its first 128-byte line in a box
    float *scores = scores_all + hl * kTile * G;

    // Sequences without tiles (length 0 or invalid) get a zero output.
    for (int b = blockIdx.x; b < p.num_seqs; b += total_ctas) {
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
    if (p.mode == 0 && blockIdx.x == 0 && warp == 0 && lane == 0)
        *p.total_tiles = total;

    using Math =
        typename std::conditional<MMA, MmaMath<D, G, TR16>, SimtMath<T, D, G, TR16>>::type;
    Math math;
    int segS = 0;          // global index of the current segment's first tile
    bool seg_bad = false;

    for (int i = R0; i < R1; ++i) {
        const int k = i - R0;
        const int s = k % spw;
        if (!ptx::mbar_wait_bounded(full0 + 8u * s, (uint32_t)((k / spw) & 1), kWaitLimitNs)) {
            if (lane == 0)
                report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
            break;
        }
        const StageMeta d = meta[s];
        const bool newseg = d.j == 0 || i == R0;
        const uint32_t kreg = sbase + (uint32_t)(s * geo.stage_bytes);
        const uint32_t vreg = kreg + (uint32_t)geo.kv_bytes;
        const uint8_t *qslot = sgen + s * geo.stage_bytes + geo.q_off + hl * geo.q_head_bytes;
        if (newseg) {
            segS = i - d.j;
            seg_bad = false;
            if constexpr (MMA)
                math.begin(qslot, lane);
            else
                math.begin(qslot, lane, p.scale_log2);
            if (p.mode == 0 && d.j == 0 && hl == 0 && lane == 0)
                p.seg_start[(int64_t)d.b * HG + d.hg] = i;
        }
        if (d.bad)
            seg_bad = true;
        if (!seg_bad) {
            if (d.n < kTile) {
                // rows past the sequence end hold whatever the pool has there:
                // zero them in this head's V (their weight is 0, but 0 * NaN is NaN)
                constexpr int NCH = D * (int)sizeof(T) / 128;
                const int lines = (kTile - d.n) * NCH;
                for (int idx = lane; idx < lines * 8; idx += 32) {
                    const int line = idx >> 3;
                    const int t = d.n + line / NCH;
                    const int ch = line % NCH;
                    const uint32_t a = tile_addr<TR16>(vreg, hline, t, ch * 8 + (idx & 7), geo);
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0)
                                 : "memory");
                }
                __syncwarp();
            }
            if constexpr (MMA)
                math.tile(kreg, vreg, hline, d.n, p.scale_log2, geo, lane);
            else
                math.tile(kreg, vreg, hline, d.n, scores, geo, lane);
        }
        // the stage may be refilled: order this warp's shared-memory accesses
        // before the producer's next TMA into it, then release it
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0)
            ptx::mbar_arrive(empty0 + 8u * s);

        // ---- end of a segment (or of this CTA's range)
        if (d.j == d.ns - 1 || i == R1 - 1) {
            math.finish();
            const int segE = segS + d.ns;
            const bool complete = segS >= R0 && segE <= R1;
            if (seg_bad && lane == 0)
                report(p.dev_status, PA_DEV_BAD_BLOCK);
            const int64_t bh0 = (int64_t)d.b * Hq + (int64_t)(d.hg * hpc + hl) * G;
            if (p.mode == 0 && !complete) {
                const int slot = ((segS < R0 ? 2 * blockIdx.x : 2 * blockIdx.x + 1) * hpc) + hl;
                float *ps = p.wpart + (int64_t)slot * p.slot_floats;
                math.for_each(
                    lane, [&](int hh, int e, float v, float) { ps[hh * D + e] = v; },
                    [&](int hh, float mm, float ll) {
                        ps[G * D + hh] = mm;
                        ps[G * D + G + hh] = ll;
                    });
                if (lane == 0)
                    ps[G * D + 2 * G] = seg_bad ? 1.f : 0.f;
            } else {
                const bool single = num_parts(d.ctx, p.partition_size) == 1;
                math.for_each(
                    lane,
                    [&](int hh, int e, float v, float ll) {
                        const float res = (seg_bad || !(ll > 0.f)) ? 0.f : v / ll;
                        if (p.public_partials)
                            p.tmp_out[((bh0 + hh) * p.max_parts + d.part) * D + e] = res;
                        if (single)
                            store_out<T>(static_cast<T *>(p.out) + (bh0 + hh) * D + e, res);
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
    }
}

// =====================================================================
// Merge of cut segments (mode 0): one CTA of merge_warps() warps per
// (sequence, KV head).  CTA x's range starts at tile floor(x T / C); the pieces
// of segment [S, S + nt) are in slot pair 2 xf + 1 of its first CTA xf and
// slot pair 2 x of every later non-empty CTA x <= xl (slot = pair * hpc +
// head within the group).  Each warp of this CTA accumulates a strided subset
// of the pieces for all G*D outputs (independent loads, so the latency is a
// few round trips whatever the piece count); the warps' sums are then added
// in shared memory.
// =====================================================================
template <int G, int D>
__host__ __device__ constexpr int merge_warps() { return G * D <= 1024 ? 8 : 4; }

template <typename T, int D, int G>
__global__ void __launch_bounds__(32 * merge_warps<G, D>()) merge_kernel(const MergeParams p)
{
    constexpr int kMergeWarps = merge_warps<G, D>();
    __shared__ float s_max[G];
    __shared__ float s_l[kMergeWarps][G];
    __shared__ float s_o[kMergeWarps][G * D];
    __shared__ int s_bad;
    const int seg = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = seg / p.num_kv_heads;
    const int h = seg - b * p.num_kv_heads;
    const int hg = h / p.hpc, hl = h - hg * p.hpc;
    const int ctx = eff_ctx(p.context_lens[b], p.ctx_cap);
    if (ctx <= 0)
        return;   // the decode kernel wrote zeros
    const int nt = ntiles(ctx);
    const int S = p.seg_start[(int64_t)b * (p.num_kv_heads / p.hpc) + hg];
    const int64_t tot = *p.total_tiles;
    const int64_t NW = p.total_ctas;
    const int wf = (int)((((int64_t)S + 1) * NW - 1) / tot);
    const int wl = (int)((((int64_t)S + nt) * NW - 1) / tot);
    if (wf == wl)
        return;   // finished inside one CTA
    // CTAs with an empty range (more CTAs than tiles) hold no piece
    auto empty = [&](int w) { return (int64_t)w * tot / NW == ((int64_t)w + 1) * tot / NW; };
    auto slot_of = [&](int w) { return (w == wf ? 2 * w + 1 : 2 * w) * p.hpc + hl; };
    const int npieces = wl - wf + 1;

    // pass 1: maxima and the bad flag
    if (threadIdx.x < G)
        s_max[threadIdx.x] = -INFINITY;
    if (threadIdx.x == 0)
        s_bad = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < npieces; i += blockDim.x) {
        const int w = wf + i;
        if (empty(w))
            continue;
        const float *ps = p.wpart + (int64_t)slot_of(w) * p.slot_floats;
        if (ps[G * D + 2 * G] != 0.f)
            atomicOr(&s_bad, 1);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mw = ps[G * D + g];
            // float max through the int ordering of non-negative / negative halves
            if (mw > -INFINITY) {
                float cur = s_max[g];
                while (mw > cur) {
                    const int old = atomicCAS(reinterpret_cast<int *>(&s_max[g]), __float_as_int(cur),
                                              __float_as_int(mw));
                    if (old == __float_as_int(cur))
                        break;
                    cur = __int_as_float(old);
                }
            }
        }
    }
    __syncthreads();
    const bool bad = s_bad != 0;

    // pass 2: warp `warp` sums pieces warp, warp + kMergeWarps, ...
    float o[G * D / 32];
    float lsum[G];
#pragma unroll
    for (int i = 0; i < G * D / 32; ++i)
        o[i] = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g)
        lsum[g] = 0.f;
    if (!bad) {
        for (int i = warp; i < npieces; i += kMergeWarps) {
            const int w = wf + i;
            if (empty(w))
                continue;
            const float *ps = p.wpart + (int64_t)slot_of(w) * p.slot_floats;
            float f[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float mw = ps[G * D + g];
                f[g] = (mw == -INFINITY || s_max[g] == -INFINITY) ? 0.f : ptx::ex2(mw - s_max[g]);
                lsum[g] = fmaf(ps[G * D + G + g], f[g], lsum[g]);
            }
#pragma unroll
            for (int i2 = 0; i2 < G * D / 32; ++i2) {
                const int idx = i2 * 32 + lane;
                o[i2] = fmaf(ps[idx], f[idx / D], o[i2]);
            }
        }
    }
#pragma unroll
    for (int i2 = 0; i2 < G * D / 32; ++i2)
        s_o[warp][i2 * 32 + lane] = o[i2];
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
            s_l[warp][g] = lsum[g];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int g = idx / D;
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kMergeWarps; ++w) {
            L += s_l[w][g];
            O += s_o[w][idx];
        }
        const int64_t bh = (int64_t)b * p.num_q_heads + (int64_t)h * G + g;
        store_out<T>(static_cast<T *>(p.out) + bh * D + (idx - g * D),
                     (!bad && L > 0.f) ? O / L : 0.f);
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
