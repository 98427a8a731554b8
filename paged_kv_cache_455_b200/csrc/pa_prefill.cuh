// pa_prefill.cuh -- sm_100a chunked-prefill paged attention: a chunk of query
// tokens per sequence attends, causally, to the sequence's cached tokens
// through its block table ("vLLM Architecture, Memory and Benchmarks Deep
// Dive", section 4, chunked prefill; section 2, block table).  bf16 data,
// fp32 accumulation on the tensor cores (mma.sync m16n8k16).
//
// One CTA per (sequence, KV head, block of query tokens).  Its 128 query rows
// are (token, query head of the group) pairs, 16 per warp, so one K/V tile
// serves every query head of the group.  A ring of stages holds 32-token K
// and V tiles of the CTA's KV head, brought by 4-D TMA boxes of min(16, bs)
// rows (one block-table entry per box) and completed on a per-stage
// mbarrier; thread 0 keeps stages - 1 tiles in flight.  Per tile each warp
// computes S = Q K^T (16 rows x 32 tokens), masks keys past each row's
// position, updates the online softmax (log2 domain, fp32), and adds P V into
// its 16 x d accumulator, P staying in registers as the A operand.
#pragma once

#include "pa_kernels.cuh"

namespace pa {

constexpr int kPfWarps = 8;
constexpr int kPfThreads = 32 * kPfWarps;
constexpr int kPfRows = 16 * kPfWarps;     // query rows per CTA
constexpr int kPfTile = 32;                // KV tokens per stage
constexpr int kPfMaxStages = 4;
constexpr int kPfMaxBlocks = 2048;         // block-table entries a CTA stages

struct PrefillParams {
    void *out;
    const void *q;
    const int32_t *cu_q_lens;
    const int32_t *block_tables;
    const int32_t *context_lens;
    int32_t *dev_status;
    int64_t num_blocks;
    int total_q;
    int num_q_heads;
    int num_kv_heads;
    int max_blocks;
    int block_size;
    int bs_log2;
    int tr;              // rows per TMA box: min(16, block_size)
    int tr_log2;
    int ctx_cap;         // lengths above this are invalid
    int qblocks;         // CTAs per (sequence, KV head)
    int stages;
    int box_stride;      // bytes between boxes (1024-aligned)
    float scale_log2;
};

// Bytes of one box of `tr` rows of one head, and its 1024-aligned stride.
__host__ __device__ constexpr int prefill_box_stride(int tr, int D)
{
    return ((tr * D * 2) + 1023) & ~1023;
}

// K and V of one 32-token tile.
__host__ __device__ constexpr int prefill_stage_bytes(int tr, int D)
{
    return 2 * (kPfTile / tr) * prefill_box_stride(tr, D);
}

// Dynamic shared memory besides the stages: alignment slack, the query rows,
// the stage barriers and the staged block-table entries.
__host__ __device__ constexpr int prefill_fixed_bytes(int D)
{
    return 1024 + kPfRows * D * 2 + 8 * kPfMaxStages + 4 * kPfMaxBlocks;
}

// 16-byte unit u of token row t of a K or V tile starting at `base`: boxes of
// tr rows, each [128-byte column][row][128 B] with the 128-byte swizzle.
__device__ __forceinline__ uint32_t pf_kv_addr(uint32_t base, int t, int u, const PrefillParams &p)
{
    const uint32_t line = (uint32_t)((u >> 3) * p.tr + (t & (p.tr - 1)));
    return base + (uint32_t)((t >> p.tr_log2) * p.box_stride) + line * 128u +
           ((((uint32_t)u & 7u) ^ (line & 7u)) << 4);
}

// 16-byte unit u of query row r ([rows][D] bf16, units XOR-swizzled by row).
template <int D>
__device__ __forceinline__ uint32_t pf_q_addr(uint32_t qbase, int r, int u)
{
    return qbase + (uint32_t)(r * D * 2) + ((((uint32_t)u) ^ ((uint32_t)r & 7u)) << 4);
}

template <int D, int G>
__device__ __forceinline__ void prefill_zero_rows(const PrefillParams &p, int q0, int tok0, int ntok,
                                                  int h)
{
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
    for (int idx = threadIdx.x; idx < ntok * G * D; idx += kPfThreads) {
        const int tok = idx / (G * D), rest = idx - tok * G * D;
        out[((int64_t)(q0 + tok0 + tok) * p.num_q_heads + h * G) * D + rest] = __float2bfloat16_rn(0.f);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p)
{
    static_assert(G >= 1 && G <= 16 && 16 % G == 0, "a warp's 16 rows hold whole tokens");
    constexpr int TQ = kPfRows / G;   // query tokens per CTA
    constexpr int KS = D / 16;        // k-steps of S over d
    constexpr int NU = D / 8;         // 16-byte units per row
    constexpr int NT = D / 8;         // n8 tiles of the accumulator over d
    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sgen = smem_raw + (sbase - raw);
    const int stages = p.stages;
    const int sbytes = 2 * (kPfTile / p.tr) * p.box_stride;
    const uint32_t qbase = sbase + (uint32_t)(stages * sbytes);
    const uint32_t bar0 = qbase + (uint32_t)(kPfRows * D * 2);
    int *sblk = reinterpret_cast<int *>(sgen + stages * sbytes + kPfRows * D * 2 + 8 * kPfMaxStages);

    const int qb = blockIdx.x % p.qblocks;
    const int rest = blockIdx.x / p.qblocks;
    const int h = rest % p.num_kv_heads;
    const int b = rest / p.num_kv_heads;

    ptx::grid_wait_prerequisites();
    const int q0 = p.cu_q_lens[b];
    const int n = p.cu_q_lens[b + 1] - q0;
    const int ctx = p.context_lens[b];
    const int tok0 = qb * TQ;
    const bool rows_ok = n >= 0 && q0 >= 0 && (int64_t)q0 + n <= p.total_q;
    if (!rows_ok || n > ctx || ctx > p.ctx_cap) {
        if (tid == 0 && qb == 0 && h == 0)
            report(p.dev_status, PA_DEV_BAD_CONTEXT);
        if (rows_ok && tok0 < n)
            prefill_zero_rows<D, G>(p, q0, tok0, min(TQ, n - tok0), h);
        return;
    }
    if (tok0 >= n)
        return;
    const int ntok = min(TQ, n - tok0);
    const int pos0 = ctx - n + tok0;                  // position of the block's first token
    const int ntiles = (pos0 + ntok - 1) / kPfTile + 1;
    const int nblk = (min(ntiles * kPfTile, ctx) - 1) / p.block_size + 1;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s)
            ptx::mbar_init(bar0 + 8u * s, 1);
    }
    ptx::fence_mbar_init();
    bool bad = false;
    const int32_t *trow = p.block_tables + (int64_t)b * p.max_blocks;
    for (int i = tid; i < nblk; i += kPfThreads) {
        const int id = trow[i];
        bad |= id < 0 || (int64_t)id >= p.num_blocks;
        sblk[i] = id;
    }
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);
    for (int idx = tid; idx < kPfRows * NU; idx += kPfThreads) {
        const int r = idx / NU, u = idx - r * NU;
        const int tok = r / G, g = r - tok * G;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (tok < ntok)
            v = *reinterpret_cast<const uint4 *>(
                qg + ((int64_t)(q0 + tok0 + tok) * p.num_q_heads + h * G + g) * D + u * 8);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(pf_q_addr<D>(qbase, r, u)),
                     "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                     : "memory");
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0)
            report(p.dev_status, PA_DEV_BAD_BLOCK);
        prefill_zero_rows<D, G>(p, q0, tok0, ntok, h);
        return;
    }

    const uint64_t policy = ptx::policy_evict_normal();
    const int boxes = kPfTile / p.tr;
    auto issue = [&](int j) {           // tile j into stage j % stages (thread 0)
        const int s = j % stages;
        const uint32_t st = sbase + (uint32_t)(s * sbytes);
        const uint32_t bar = bar0 + 8u * s;
        int nbox = 0;
        while (nbox < boxes && j * kPfTile + nbox * p.tr < ctx)
            ++nbox;
        ptx::mbar_arrive_expect_tx(bar, (uint32_t)(2 * nbox * p.tr * D * 2));
        for (int k = 0; k < nbox; ++k) {
            const int t = j * kPfTile + k * p.tr;
            const int row = sblk[t >> p.bs_log2] * p.block_size + (t & (p.block_size - 1));
            ptx::tma_load_4d(st + (uint32_t)(k * p.box_stride), &tmap_k, 0, row, 0, h, bar, policy);
            ptx::tma_load_4d(st + (uint32_t)((boxes + k) * p.box_stride), &tmap_v, 0, row, 0, h, bar,
                             policy);
        }
    };
    if (tid == 0) {
        ptx::prefetch_tensormap(&tmap_k);
        ptx::prefetch_tensormap(&tmap_v);
        for (int j = 0; j < stages - 1 && j < ntiles; ++j)
            issue(j);
    }

    const int ra = warp * 16 + (lane >> 2), rb = ra + 8;   // this lane's two rows
    const int pa_ = pos0 + ra / G, pb_ = pos0 + rb / G;     // their positions
    float o[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
        o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;
    int j = 0;
    for (; j < ntiles; ++j) {
        if (tid == 0 && j + stages - 1 < ntiles)
            issue(j + stages - 1);
        const int s = j % stages;
        const bool arrived = ptx::mbar_wait_bounded(bar0 + 8u * s, (uint32_t)((j / stages) & 1),
                                                    kWaitLimitNs);
        const uint32_t kb = sbase + (uint32_t)(s * sbytes);
        const uint32_t vb = kb + (uint32_t)(boxes * p.box_stride);
        const int tstart = j * kPfTile;
        if (tstart + kPfTile > ctx) {
            // rows past the context: whatever the pool or an older tile left
            // there; their weight is 0, but 0 * NaN is NaN, so zero them in V
            const int from = ctx - tstart;
            for (int idx = tid; idx < (kPfTile - from) * NU; idx += kPfThreads) {
                const int t = from + idx / NU, u = idx % NU;
                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(pf_kv_addr(vb, t, u, p)),
                             "r"(0)
                             : "memory");
            }
            __syncthreads();
        }
        // ---- S = Q K^T: 16 rows x 32 tokens
        float sc[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            sc[t][0] = sc[t][1] = sc[t][2] = sc[t][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            uint32_t a[4];
            ptx::ldsm_x4(pf_q_addr<D>(qbase, warp * 16 + (lane & 15), 2 * kk + (lane >> 4)), a);
#pragma unroll
            for (int np2 = 0; np2 < 2; ++np2) {
                uint32_t bb[4];
                ptx::ldsm_x4(pf_kv_addr(kb, 16 * np2 + (lane & 7) + ((lane >> 4) << 3),
                                        2 * kk + ((lane >> 3) & 1), p),
                             bb);
                ptx::mma_bf16_16816(sc[2 * np2], a, bb[0], bb[1]);
                ptx::mma_bf16_16816(sc[2 * np2 + 1], a, bb[2], bb[3]);
            }
        }
        // ---- causal mask and online softmax (rows ra: elements 0, 1; rb: 2, 3)
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int key = tstart + 8 * t + 2 * (lane & 3);
            sc[t][0] = key <= pa_ ? sc[t][0] * p.scale_log2 : -INFINITY;
            sc[t][1] = key + 1 <= pa_ ? sc[t][1] * p.scale_log2 : -INFINITY;
            sc[t][2] = key <= pb_ ? sc[t][2] * p.scale_log2 : -INFINITY;
            sc[t][3] = key + 1 <= pb_ ? sc[t][3] * p.scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(sc[t][0], sc[t][1]));
            mx1 = fmaxf(mx1, fmaxf(sc[t][2], sc[t][3]));
        }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = mn0 == -INFINITY ? 1.f : ptx::ex2(m0 - mn0);
        const float al1 = mn1 == -INFINITY ? 1.f : ptx::ex2(m1 - mn1);
        const float rf0 = mn0 == -INFINITY ? 0.f : mn0;
        const float rf1 = mn1 == -INFINITY ? 0.f : mn1;
        m0 = mn0;
        m1 = mn1;
        uint32_t pa[2][4];
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int t = 2 * ks + half;
                const uint32_t lo = ptx::pack_bf16x2(ptx::ex2(sc[t][0] - rf0), ptx::ex2(sc[t][1] - rf0));
                const uint32_t hi = ptx::pack_bf16x2(ptx::ex2(sc[t][2] - rf1), ptx::ex2(sc[t][3] - rf1));
                // the sums use the same rounded weights as the MMA
                ps0 += ptx::bf16lo_to_f32(lo) + ptx::bf16hi_to_f32(lo);
                ps1 += ptx::bf16lo_to_f32(hi) + ptx::bf16hi_to_f32(hi);
                pa[ks][2 * half] = lo;
                pa[ks][2 * half + 1] = hi;
            }
        }
        l0 = l0 * al0 + ps0;
        l1 = l1 * al1 + ps1;
        if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                o[t][0] *= al0;
                o[t][1] *= al0;
                o[t][2] *= al1;
                o[t][3] *= al1;
            }
        }
        // ---- O += P V: 16 rows x d, k over the 32 tokens
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
            for (int jp = 0; jp < NT / 2; ++jp) {
                uint32_t bb[4];
                ptx::ldsm_x4_trans(pf_kv_addr(vb, 16 * ks + (lane & 7) + (((lane >> 3) & 1) << 3),
                                              2 * jp + (lane >> 4), p),
                                   bb);
                ptx::mma_bf16_16816(o[2 * jp], pa[ks], bb[0], bb[1]);
                ptx::mma_bf16_16816(o[2 * jp + 1], pa[ks], bb[2], bb[3]);
            }
        }
        // the stage may be refilled after the barrier: order this thread's
        // shared-memory accesses before the next TMA into it
        ptx::fence_proxy_async_smem();
        if (!__syncthreads_and(arrived)) {
            ok = false;
            break;
        }
    }
    if (!ok) {
        // a copy never arrived: let every issued copy land (bounded), then stop
        if (tid == 0) {
            report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
            for (int i = j; i < min(ntiles, j + stages - 1) + 1 && i < ntiles; ++i)
                ptx::mbar_wait_bounded(bar0 + 8u * (i % stages), (uint32_t)((i / stages) & 1),
                                       kWaitLimitNs);
        }
        __syncthreads();
        return;
    }

    // ---- normalise and store (bf16 pairs of consecutive d)
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, off);
        l1 += __shfl_xor_sync(kFull, l1, off);
    }
    const float i0 = l0 > 0.f ? __frcp_rn(l0) : 0.f;
    const float i1 = l1 > 0.f ? __frcp_rn(l1) : 0.f;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
    const int c2 = 2 * (lane & 3);
    if (ra / G < ntok) {
        uint32_t *dst = reinterpret_cast<uint32_t *>(
            out + ((int64_t)(q0 + tok0 + ra / G) * p.num_q_heads + h * G + ra % G) * D + c2);
#pragma unroll
        for (int t = 0; t < NT; ++t)
            dst[4 * t] = ptx::pack_bf16x2(o[t][0] * i0, o[t][1] * i0);
    }
    if (rb / G < ntok) {
        uint32_t *dst = reinterpret_cast<uint32_t *>(
            out + ((int64_t)(q0 + tok0 + rb / G) * p.num_q_heads + h * G + rb % G) * D + c2);
#pragma unroll
        for (int t = 0; t < NT; ++t)
            dst[4 * t] = ptx::pack_bf16x2(o[t][2] * i1, o[t][3] * i1);
    }
}

}  // namespace pa
