// pa_prefill_tc.cuh -- chunked-prefill paged attention on the 5th-generation
// tensor cores (tcgen05.mma, accumulators in tensor memory), for block sizes
// of 16 and 32 ("vLLM Architecture, Memory and Benchmarks Deep Dive",
// section 4, chunked prefill; section 2, block table).  Same contract as the
// mma.sync kernel in pa_prefill.cuh.
//
// One CTA per (sequence, KV head, 128 query rows); row r is (token r / G,
// query head r % G of the group), so one K/V tile serves the whole group.
// Warps 0-3 own one query row per thread; warp 4 is the control warp.
//
//   control (one thread)            TMA: Q once; K and V of 64-token tiles
//                                   into two stages (16-row boxes of one KV
//                                   head, 128-byte swizzle)
//                                   S_j = Q K_j^T: 4 x 16 MMAs of M=128,N=16,
//                                   K=16 into S buffer j % 2 (TMEM, fp32)
//                                   O += P_j V_j: 4 MMAs of M=128, N=d, K=16,
//                                   V read MN-major straight from its boxes
//   softmax (128 threads)           S row from TMEM (tcgen05.ld), causal
//                                   mask, running max; O rescaled in TMEM
//                                   only when the max grew by more than 2^8;
//                                   P = 2^(s - m) to shared memory (bf16,
//                                   swizzled K-major), row sum in fp32
//
// Completion is tracked by mbarriers: TMA tx counts for the stages, and
// tcgen05.commit for the MMAs.  Every wait is bounded; a timeout stops all
// warps through a shared flag, and the tensor memory is released on every
// path.
#pragma once

#include "pa_prefill.cuh"

namespace pa {

constexpr int kTcRows = 128;            // query rows per CTA (MMA M)
constexpr int kTcTile = 64;             // KV tokens per stage
constexpr int kTcBoxes = kTcTile / 16;  // 16-row boxes per K or V tile
constexpr int kTcThreads = 160;         // 4 softmax warps + 1 control warp

// Shared memory layout (bytes from the 1024-aligned base), per head dim.
__host__ __device__ constexpr int tc_box_bytes(int D) { return 16 * D * 2; }
__host__ __device__ constexpr int tc_q_bytes(int D) { return kTcRows * D * 2; }
__host__ __device__ constexpr int tc_stage_bytes(int D) { return 2 * kTcBoxes * tc_box_bytes(D); }
__host__ __device__ constexpr int tc_p_off(int D) { return tc_q_bytes(D) + 2 * tc_stage_bytes(D); }
__host__ __device__ constexpr int tc_blk_off(int D) { return tc_p_off(D) + kTcRows * 128; }
__host__ __device__ constexpr int tc_bar_off(int D) { return tc_blk_off(D) + 4 * kPfMaxBlocks; }
__host__ __device__ constexpr int tc_smem_bytes(int D) { return 1024 + tc_bar_off(D) + 128; }
__host__ __device__ constexpr uint32_t tc_tmem_cols(int D) { return 128 + D <= 256 ? 256u : 512u; }

template <int D, int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p)
{
    static_assert(D % 64 == 0 && D <= 256, "head dim of 64, 128 or 256");
    static_assert(G >= 1 && 128 % G == 0, "whole tokens per CTA");
    constexpr int TQ = kTcRows / G;
    constexpr int NCH = D / 64;                   // 128-byte columns per row
    constexpr int BOX = tc_box_bytes(D);
    constexpr uint32_t TCOLS = tc_tmem_cols(D);
    constexpr uint32_t IDESC_S = ptx::umma_idesc_bf16(128, 16, false, false);
    constexpr uint32_t IDESC_O = ptx::umma_idesc_bf16(128, D, false, true);

    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t q_s = base;
    const uint32_t stage_s = base + tc_q_bytes(D);
    const uint32_t p_s = base + tc_p_off(D);
    int *sblk = reinterpret_cast<int *>(gbase + tc_blk_off(D));
    const uint32_t bars = base + tc_bar_off(D);
    // barriers: full[2], empty[2], sfull[2], pready, odone, qfull
    const uint32_t full0 = bars, empty0 = bars + 16, sfull0 = bars + 32, pready = bars + 48,
                   odone = bars + 56, qfull = bars + 64;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gbase + tc_bar_off(D) + 72);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + tc_bar_off(D) + 76);

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
        if (rows_ok && tok0 < n) {
            __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
            const int nt = min(TQ, n - tok0);
            for (int idx = tid; idx < nt * G * D; idx += kTcThreads) {
                const int tok = idx / (G * D), r = idx - tok * G * D;
                out[((int64_t)(q0 + tok0 + tok) * p.num_q_heads + h * G) * D + r] =
                    __float2bfloat16_rn(0.f);
            }
        }
        return;
    }
    if (tok0 >= n)
        return;
    const int ntok = min(TQ, n - tok0);
    const int pos0 = ctx - n + tok0;
    const int ntiles = (pos0 + ntok - 1) / kTcTile + 1;
    const int nblk = (min(ntiles * kTcTile, ctx) - 1) / p.block_size + 1;

    // ---- set-up: barriers, block ids, tensor memory
    if (tid == 0) {
        ptx::mbar_init(full0, 1);
        ptx::mbar_init(full0 + 8, 1);
        ptx::mbar_init(empty0, 1);
        ptx::mbar_init(empty0 + 8, 1);
        ptx::mbar_init(sfull0, 1);
        ptx::mbar_init(sfull0 + 8, 1);
        ptx::mbar_init(pready, 4);
        ptx::mbar_init(odone, 1);
        ptx::mbar_init(qfull, 1);
        *abort_flag = 0;
    }
    ptx::fence_mbar_init();
    bool bad = false;
    const int32_t *trow = p.block_tables + (int64_t)b * p.max_blocks;
    for (int i = tid; i < nblk; i += kTcThreads) {
        const int id = trow[i];
        bad |= id < 0 || (int64_t)id >= p.num_blocks;
        sblk[i] = id;
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_holder), TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    bad = __syncthreads_or(bad);
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t s_tm = tmem;            // S buffers: columns [0, 64) and [64, 128)
    const uint32_t o_tm = tmem + 128;      // O: columns [128, 128 + D)

    if (bad) {
        if (tid == 0)
            report(p.dev_status, PA_DEV_BAD_BLOCK);
    } else if (warp == 4) {
        // ================================================ control warp
        if (lane == 0) {
            auto issue_kv = [&](int j) {
                const int s = j & 1;
                const uint32_t kst = stage_s + (uint32_t)(s * tc_stage_bytes(D));
                const uint32_t vst = kst + (uint32_t)(kTcBoxes * BOX);
                int nbox = 0;
                while (nbox < kTcBoxes && j * kTcTile + nbox * 16 < ctx)
                    ++nbox;
                ptx::mbar_arrive_expect_tx(full0 + 8u * s, (uint32_t)(2 * nbox * BOX));
                for (int k = 0; k < nbox; ++k) {
                    const int t = j * kTcTile + k * 16;
                    const int row = sblk[t >> p.bs_log2] * p.block_size + (t & (p.block_size - 1));
                    ptx::tma_load_4d(kst + (uint32_t)(k * BOX), &tmap_k, 0, row, 0, h, full0 + 8u * s,
                                     ptx::policy_evict_normal());
                    ptx::tma_load_4d(vst + (uint32_t)(k * BOX), &tmap_v, 0, row, 0, h, full0 + 8u * s,
                                     ptx::policy_evict_normal());
                }
            };
            auto issue_s = [&](int j) {        // S_j = Q K_j^T into buffer j & 1
                const uint32_t kst = stage_s + (uint32_t)((j & 1) * tc_stage_bytes(D));
                for (int box = 0; box < kTcBoxes; ++box)
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = ptx::umma_desc_sw128(
                            q_s + (uint32_t)((kk >> 2) * kTcRows * 128 + (kk & 3) * 32), 16, 1024);
                        const uint64_t bd = ptx::umma_desc_sw128(
                            kst + (uint32_t)(box * BOX + (kk >> 2) * 2048 + (kk & 3) * 32), 16,
                            1024);
                        ptx::umma_bf16_ss(s_tm + (uint32_t)((j & 1) * 64 + box * 16), a, bd,
                                          IDESC_S, kk > 0);
                    }
                ptx::umma_commit(sfull0 + 8u * (j & 1));
            };
            bool ok = true;
            ptx::prefetch_tensormap(&tmap_q);
            ptx::prefetch_tensormap(&tmap_k);
            ptx::prefetch_tensormap(&tmap_v);
            ptx::mbar_arrive_expect_tx(qfull, (uint32_t)tc_q_bytes(D));
            for (int c = 0; c < NCH; ++c)
                ptx::tma_load_3d_nohint(q_s + (uint32_t)(c * kTcRows * 128), &tmap_q, c * 64,
                                        h * G, q0 + tok0, qfull);
            issue_kv(0);
            if (ntiles > 1)
                issue_kv(1);
            ok = ptx::mbar_wait_bounded(qfull, 0, kWaitLimitNs) &&
                 ptx::mbar_wait_bounded(full0, 0, kWaitLimitNs);
            if (ok) {
                ptx::tc_fence_after();
                issue_s(0);
            }
            for (int j = 0; ok && j < ntiles; ++j) {
                if (*abort_flag)
                    break;
                if (j + 1 < ntiles) {
                    ok = ptx::mbar_wait_bounded(full0 + 8u * ((j + 1) & 1),
                                                (uint32_t)(((j + 1) >> 1) & 1), kWaitLimitNs);
                    if (!ok)
                        break;
                    ptx::tc_fence_after();
                    issue_s(j + 1);
                }
                ok = ptx::mbar_wait_bounded(pready, (uint32_t)(j & 1), kWaitLimitNs);
                if (!ok)
                    break;
                ptx::tc_fence_after();
                const uint32_t vst =
                    stage_s + (uint32_t)((j & 1) * tc_stage_bytes(D) + kTcBoxes * BOX);
                for (int box = 0; box < kTcBoxes; ++box) {
                    const uint64_t a = ptx::umma_desc_sw128(p_s + (uint32_t)(box * 32), 16, 1024);
                    const uint64_t bd =
                        ptx::umma_desc_sw128(vst + (uint32_t)(box * BOX), 2048, 1024);
                    ptx::umma_bf16_ss(o_tm, a, bd, IDESC_O, j > 0 || box > 0);
                }
                ptx::umma_commit(empty0 + 8u * (j & 1));
                ptx::umma_commit(odone);
                if (j + 2 < ntiles) {
                    ok = ptx::mbar_wait_bounded(empty0 + 8u * (j & 1), (uint32_t)((j >> 1) & 1),
                                                kWaitLimitNs);
                    if (!ok)
                        break;
                    issue_kv(j + 2);
                }
            }
            if (!ok) {
                report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
        }
        __syncwarp();
    } else {
        // ================================================ softmax warps
        const int r = tid;                          // query row = TMEM lane
        const int pos = pos0 + r / G;
        const uint32_t lane_tm = (uint32_t)(warp * 32) << 16;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        // tcgen05.ld / st / wait are .sync.aligned: every decision that
        // guards one is made for the whole warp
        for (int j = 0; j < ntiles; ++j) {
            if (__any_sync(kFull, *abort_flag != 0)) {
                ok = false;
                break;
            }
            if (!__all_sync(kFull, ptx::mbar_wait_bounded(sfull0 + 8u * (j & 1),
                                                          (uint32_t)((j >> 1) & 1),
                                                          kWaitLimitNs))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            float sv[kTcTile];
#pragma unroll
            for (int c = 0; c < kTcTile / 16; ++c) {
                uint32_t u[16];
                ptx::tmem_ld16(s_tm + lane_tm + (uint32_t)((j & 1) * 64 + c * 16), u);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    sv[c * 16 + e] = __uint_as_float(u[e]);
            }
            const int tstart = j * kTcTile;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kTcTile; ++c) {
                sv[c] = tstart + c <= pos ? sv[c] * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, sv[c]);
            }
            if (j > 0) {
                // the previous P V is done: P may be overwritten, O is stable
                if (!__all_sync(kFull, ptx::mbar_wait_bounded(odone, (uint32_t)((j - 1) & 1),
                                                              kWaitLimitNs))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
            }
            bool grow = false;
            float alpha = 1.f;
            if (m_ref == -INFINITY) {
                m_ref = mx;                          // nothing accumulated yet
            } else if (mx > m_ref + 8.f) {
                grow = true;
                alpha = ptx::ex2(m_ref - mx);
            }
            if (__any_sync(kFull, grow)) {
                // the whole warp rescales its rows of O (alpha = 1 for rows
                // whose max did not grow)
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t u[16];
                    ptx::tmem_ld16(o_tm + lane_tm + (uint32_t)(c * 16), u);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
                    ptx::tmem_st16(o_tm + lane_tm + (uint32_t)(c * 16), u);
                }
                ptx::tmem_wait_st();
            }
            if (grow) {
                l *= alpha;
                m_ref = mx;
            }
            const float ref = m_ref == -INFINITY ? 0.f : m_ref;
            // P row: 64 bf16 = 8 16-byte units, unit u at ((u ^ (r & 7)) << 4)
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                uint32_t w[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t pk = ptx::pack_bf16x2(ptx::ex2(sv[8 * u + 2 * k] - ref),
                                                         ptx::ex2(sv[8 * u + 2 * k + 1] - ref));
                    l += ptx::bf16lo_to_f32(pk) + ptx::bf16hi_to_f32(pk);
                    w[k] = pk;
                }
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                                 p_s + (uint32_t)(r * 128) + ((uint32_t)(u ^ (r & 7)) << 4)),
                             "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                             : "memory");
            }
            if (tstart + kTcTile > ctx) {
                // V rows past the context: whatever the pool or an older tile
                // left there; their weight is 0, but 0 * NaN is NaN.  (The
                // stage's copies are complete: S_j, which follows them, is.)
                if (!__all_sync(kFull, ptx::mbar_wait_bounded(full0 + 8u * (j & 1),
                                                              (uint32_t)((j >> 1) & 1),
                                                              kWaitLimitNs))) {
                    ok = false;
                    break;
                }
                const uint32_t vst =
                    stage_s + (uint32_t)((j & 1) * tc_stage_bytes(D) + kTcBoxes * BOX);
                const int from = ctx - tstart;
                for (int idx = r; idx < (kTcTile - from) * NCH * 8; idx += kTcRows) {
                    const int t = from + idx / (NCH * 8), rem = idx % (NCH * 8);
                    const uint32_t a = vst + (uint32_t)((t >> 4) * BOX + (rem >> 3) * 2048 +
                                                        (t & 15) * 128 + (rem & 7) * 16);
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0)
                                 : "memory");
                }
            }
            // the MMA reads P and V through the async proxy
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(pready);
        }
        if (ok && !__all_sync(kFull, ptx::mbar_wait_bounded(odone, (uint32_t)((ntiles - 1) & 1),
                                                            kWaitLimitNs)))
            ok = false;
        if (!ok) {
            if (lane == 0)
                report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
        } else {
            ptx::tc_fence_after();
            // ---- normalise and store this row (bf16)
            const float inv = l > 0.f ? __frcp_rn(l) : 0.f;
            const bool store = r / G < ntok;     // every lane loads; valid rows store
            uint4 *dst = reinterpret_cast<uint4 *>(
                static_cast<__nv_bfloat16 *>(p.out) +
                ((int64_t)(q0 + tok0 + (store ? r / G : 0)) * p.num_q_heads + h * G + r % G) * D);
            for (int c = 0; c < D / 16; ++c) {
                uint32_t u[16];
                ptx::tmem_ld16(o_tm + lane_tm + (uint32_t)(c * 16), u);
                ptx::tmem_wait_ld();
                uint4 a, b2;
                a.x = ptx::pack_bf16x2(__uint_as_float(u[0]) * inv, __uint_as_float(u[1]) * inv);
                a.y = ptx::pack_bf16x2(__uint_as_float(u[2]) * inv, __uint_as_float(u[3]) * inv);
                a.z = ptx::pack_bf16x2(__uint_as_float(u[4]) * inv, __uint_as_float(u[5]) * inv);
                a.w = ptx::pack_bf16x2(__uint_as_float(u[6]) * inv, __uint_as_float(u[7]) * inv);
                b2.x = ptx::pack_bf16x2(__uint_as_float(u[8]) * inv, __uint_as_float(u[9]) * inv);
                b2.y = ptx::pack_bf16x2(__uint_as_float(u[10]) * inv, __uint_as_float(u[11]) * inv);
                b2.z = ptx::pack_bf16x2(__uint_as_float(u[12]) * inv, __uint_as_float(u[13]) * inv);
                b2.w = ptx::pack_bf16x2(__uint_as_float(u[14]) * inv, __uint_as_float(u[15]) * inv);
                if (store) {
                    dst[2 * c] = a;
                    dst[2 * c + 1] = b2;
                }
            }
        }
    }
    if (bad) {
        // zero this CTA's rows
        __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
        for (int idx = tid; idx < ntok * G * D; idx += kTcThreads) {
            const int tok = idx / (G * D), rr = idx - tok * G * D;
            out[((int64_t)(q0 + tok0 + tok) * p.num_q_heads + h * G) * D + rr] =
                __float2bfloat16_rn(0.f);
        }
    }
    // ---- release the tensor memory (every tcgen05 operation is complete:
    // the last P V was waited for, or nothing was issued, or a wait gave up)
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 0)
        ptx::tmem_dealloc(tmem, TCOLS);
}

}  // namespace pa
