// pa_prefill_tc.cuh -- chunked-prefill paged attention on the 5th-generation
// tensor cores (tcgen05.mma, accumulators in tensor memory), for block sizes
// of 16 and 32 ("vLLM Architecture, Memory and Benchmarks Deep Dive",
// section 4, chunked prefill; section 2, block table).  Same contract as the
// mma.sync kernel in pa_prefill.cuh.
//
// One CTA per (sequence, KV head, 128 query rows); row r is (token r / G,
// query head r % G of the group), so one K/V tile serves the whole group.
// Warps 0-3 own one query row per thread; warp 4 issues the MMAs, warps 5
// and 6 the TMA copies of K and V (warp 7 has no work).
//
//   producers (5, 6)    TMA: Q once; K tiles into four stages, V tiles into
//                       three (one of each in the space Q held before it
//                       moved to tensor memory), one box per 16 tokens (lane k
//                       issues box k of a tile); through a 5-D map a box
//                       lands as [8-token group][128-byte column][token]
//                       [128 bytes] with 128-byte swizzle, so 8-token groups
//                       are a fixed d * 16 bytes apart across the whole tile
//   MMA (warp 4)        S_j = Q K_j^T (M=128, N=64, K=16 steps) with Q read
//                       from tensor memory and K from its stage; O += P_j V_j
//                       (M=128, N=d, K=16 per block) with P_j read from
//                       tensor memory and V MN-major straight from its stage.
//                       S_{j+1} is issued before P_{j-1} V_{j-1}, so that the
//                       softmax gets it first.  The two write disjoint tensor
//                       memory and every reuse is guarded by a barrier.  A K stage is free when its S is
//                       done, a V stage and a P buffer when their P V is
//                       (tcgen05.commit)
//   softmax (warps 0-3) first move the CTA's Q rows from shared to tensor
//                       memory; then per tile: S row from tensor memory (the
//                       S buffer is released as soon as it is read), causal
//                       mask on diagonal tiles, running max; O rescaled in
//                       tensor memory only when the max grew by more than
//                       2^8; P = 2^(s - m) as bf16 into P buffer j % 2 of
//                       tensor memory; row sum in fp32 of the fp32 weights
//
// Tensor memory columns: S [0, 64), O [64, 64 + d), Q (d / 2 columns: two
// bf16 per column) at 64 + d, P buffers (32 columns) after it.  With Q in
// tensor memory an S MMA reads only K from shared memory.  S_{j+1} and
// P_{j-1} V_{j-1} run while the softmax of tile j computes.
// Every wait is bounded; a timeout stops all warps through a shared flag,
// and the tensor memory is released on every path.
#pragma once

#include "pa_prefill.cuh"

namespace pa {

constexpr int kTcRows = 128;            // query rows per CTA (MMA M)
constexpr int kTcTile = 64;             // KV tokens per stage
constexpr int kTcBoxes = kTcTile / 16;  // 16-token blocks per tile
constexpr int kTcKStages = 4;           // three after Q, one where Q was
constexpr int kTcVStages = 3;           // two after the K stages, one where Q was
constexpr int kTcThreads = 256;         // 4 softmax warps, 2 MMA warps, 2 TMA warps

// Shared memory layout (bytes from the 1024-aligned base), per head dim:
// Q (then K stage 3, V stage 2) | K stages 0-2 | V stages 0, 1 | barriers.
// The Q region holds exactly two stages.  In a stage, column c of token t is
// at
// (t / 8) * (d * 16) + c * 1024 + (t % 8) * 128.
__host__ __device__ constexpr int tc_group_bytes(int D) { return 8 * D * 2; }
__host__ __device__ constexpr int tc_box_bytes(int D) { return 16 * D * 2; }
__host__ __device__ constexpr int tc_q_bytes(int D) { return kTcRows * D * 2; }
__host__ __device__ constexpr int tc_kv_bytes(int D) { return kTcBoxes * tc_box_bytes(D); }
__host__ __device__ constexpr int tc_bar_off(int D)
{
    return tc_q_bytes(D) + 5 * tc_kv_bytes(D);
}
__host__ __device__ constexpr int tc_smem_bytes(int D) { return 1024 + tc_bar_off(D) + 256; }
__host__ __device__ constexpr uint32_t tc_tmem_cols(int D)
{
    return 64 + D + D / 2 + 64 <= 256 ? 256u : 512u;
}

// 16-token blocks of tile j that hold tokens of a context of ctx tokens.
__device__ __forceinline__ int tc_boxes(int j, int ctx)
{
    return min(kTcBoxes, (ctx - j * kTcTile + 15) >> 4);
}

template <int D, int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p)
{
    static_assert(D % 64 == 0 && D <= 256, "head dim of 64, 128 or 256");
    static_assert(G >= 1 && 128 % G == 0, "whole tokens per CTA");
    static_assert(tc_smem_bytes(D) <= 232448, "shared memory per CTA");
    constexpr int TQ = kTcRows / G;
    constexpr int NCH = D / 64;                   // 128-byte columns per row
    constexpr int BOX = tc_box_bytes(D);
    constexpr int KV = tc_kv_bytes(D);
    constexpr uint32_t TCOLS = tc_tmem_cols(D);
    constexpr uint32_t IDESC_S = ptx::umma_idesc_bf16(128, kTcTile, false, false);
    constexpr uint32_t IDESC_O = ptx::umma_idesc_bf16(128, D, false, true);

    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t q_s = base;
    const uint32_t n_s = base + tc_q_bytes(D);            // the five stages after Q
    auto kstage = [&](int s) {                            // K stage s (3: where Q was)
        return s < 3 ? n_s + (uint32_t)(s * KV) : q_s;
    };
    auto vstage = [&](int s) {                            // V stage s (2: where Q was)
        return s < 2 ? n_s + (uint32_t)((3 + s) * KV) : q_s + (uint32_t)KV;
    };
    const uint32_t bars = base + tc_bar_off(D);
    // kfull[4], kempty[4], vfull[3], vempty[3], pready[2], pfree[2], sfull, sfree,
    // qfull, qready
    const uint32_t kfull = bars, kempty = bars + 32, vfull = bars + 64, vempty = bars + 88,
                   pready = bars + 112, pfree = bars + 128, sfull = bars + 144,
                   sfree = bars + 152, qfull = bars + 160, qready = bars + 168;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gbase + tc_bar_off(D) + 176);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + tc_bar_off(D) + 180);

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

    // ---- set-up: barriers, block-id check, tensor memory
    if (tid == 0) {
        for (int i = 0; i < kTcKStages; ++i) {
            ptx::mbar_init(kfull + 8u * i, 1);
            ptx::mbar_init(kempty + 8u * i, 1);
        }
        for (int i = 0; i < kTcVStages; ++i) {
            ptx::mbar_init(vfull + 8u * i, 1);
            ptx::mbar_init(vempty + 8u * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(pready + 8u * i, 4);
            ptx::mbar_init(pfree + 8u * i, 1);
        }
        ptx::mbar_init(sfull, 1);
        ptx::mbar_init(sfree, 4);
        ptx::mbar_init(qfull, 1);
        ptx::mbar_init(qready, 4);
        *abort_flag = 0;
    }
    ptx::fence_mbar_init();
    bool bad = false;
    const int32_t *trow = p.block_tables + (int64_t)b * p.max_blocks;
    for (int i = tid; i < nblk; i += kTcThreads) {
        const int id = trow[i];
        bad |= id < 0 || (int64_t)id >= p.num_blocks;
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_holder), TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    bad = __syncthreads_or(bad);
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t s_tm = tmem;
    const uint32_t o_tm = tmem + 64;
    const uint32_t q_tm = tmem + 64 + (uint32_t)D;
    const uint32_t p_tm = q_tm + (uint32_t)(D / 2);  // P buffer s at p_tm + 32 s

    if (bad) {
        if (tid == 0)
            report(p.dev_status, PA_DEV_BAD_BLOCK);
    } else if (warp == 5 || warp == 6) {
        // ================================================ TMA producers
        // warp 5 copies K (and Q), warp 6 copies V; lane x issues box x
        // (tokens 16 x .. 16 x + 15) of each tile
        const bool is_k = warp == 5;
        const int xb = lane;
        const uint32_t full = is_k ? kfull : vfull, empty = is_k ? kempty : vempty;
        const int nst = is_k ? kTcKStages : kTcVStages;
        const void *tmap = is_k ? static_cast<const void *>(&tmap_k)
                                : static_cast<const void *>(&tmap_v);
        bool ok = true;
        if (lane == 0) {
            ptx::prefetch_tensormap(tmap);
            if (is_k) {
                ptx::prefetch_tensormap(&tmap_q);
                ptx::mbar_arrive_expect_tx(qfull, (uint32_t)tc_q_bytes(D));
                for (int c = 0; c < NCH; ++c)
                    ptx::tma_load_3d_nohint(q_s + (uint32_t)(c * kTcRows * 128), &tmap_q, c * 64,
                                            h * G, q0 + tok0, qfull);
            }
        }
        // block ids come 32 at a time, lane l holding entry 32 * batch + l,
        // one batch ahead, so that no copy waits for the table; a tile's
        // blocks lie in one batch (a batch is 32 blocks >= 512 tokens)
        auto batch_ids = [&](int bt) {
            const int i = bt * 32 + lane;
            return i < nblk ? __ldg(trow + i) : -1;
        };
        int ids_cur = batch_ids(0), ids_next = batch_ids(1), cur_batch = 0;
        int issued = 0;
        for (int i = 0; i < ntiles; ++i) {
            if (__any_sync(kFull, *abort_flag != 0))
                break;
            const int bt = (i * kTcTile) >> (p.bs_log2 + 5);   // same for all lanes
            if (bt != cur_batch) {
                cur_batch = bt;
                ids_cur = ids_next;
                ids_next = batch_ids(bt + 1);
            }
            const int id = __shfl_sync(kFull, ids_cur, ((i * kTcTile + xb * 16) >> p.bs_log2) & 31);
            const int s = i % nst, nbox = tc_boxes(i, ctx);
            const int row = id * p.block_size + ((i * kTcTile + xb * 16) & (p.block_size - 1));
            if (i >= nst) {
                ok = __all_sync(kFull, ptx::mbar_wait_bounded(empty + 8u * s,
                                                              (uint32_t)((i / nst - 1) & 1),
                                                              kWaitLimitNs));
            } else if (s == (is_k ? 3 : 2)) {
                // the stage where Q was: wait until Q is in tensor memory
                ok = __all_sync(kFull, ptx::mbar_wait_bounded(qready, 0, kWaitLimitNs));
            }
            if (!ok)
                break;
            const uint32_t dst = is_k ? kstage(s) : vstage(s);
            if (lane == 0)
                ptx::mbar_arrive_expect_tx(full + 8u * s, (uint32_t)(nbox * BOX));
            __syncwarp();
            if (xb < nbox)
                ptx::tma_load_5d(dst + (uint32_t)(xb * BOX), tmap, 0, 0, 0, row >> 3, h,
                                 full + 8u * s, ptx::policy_evict_normal());
            issued = i + 1;
        }
        if (lane == 0) {
            if (!ok) {
                report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // no copy may land after the CTA is gone: wait (bounded) for the
            // last ones issued to each stage; on the normal path the MMA
            // thread has already seen them all
            if (is_k)
                ptx::mbar_wait_bounded(qfull, 0, kWaitLimitNs);
            for (int i = max(0, issued - nst); i < issued; ++i)
                ptx::mbar_wait_bounded(full + 8u * (i % nst), (uint32_t)((i / nst) & 1),
                                       kWaitLimitNs);
        }
        __syncwarp();
    } else if (warp == 4 || warp == 7) {
        // ================================================ MMA issue
        // Warp 4: S_0, then S_{j+1} once the softmax has read S_j out of
        // tensor memory and K_{j+1} has landed, and P_j V_j once the softmax
        // has written P_j and V_j has landed (warp 7 idles here).  The whole
        // warp waits (suspending, so it takes no issue slots from the softmax
        // warps);
        // one elected lane, always lane 0, issues the MMAs and their commits
        // (a commit tracks the MMAs of its own thread).
        // descriptors: K is K-major, 8-token groups d * 16 bytes apart; V is
        // MN-major, 64-element columns 1024 bytes apart, 8-token groups
        // d * 16 bytes apart
        // both phases complete?  One non-blocking test and one vote when
        // they are (the usual case); else suspending waits, unless another
        // warp has given up
        auto ready = [&](uint32_t b1, uint32_t p1, uint32_t b2, uint32_t p2) -> bool {
            if (__all_sync(kFull, ptx::mbar_test_wait(b1, p1) && ptx::mbar_test_wait(b2, p2)))
                return true;
            if (__any_sync(kFull, *abort_flag != 0))
                return false;
            return __all_sync(kFull, ptx::mbar_wait_bounded(b1, p1, kWaitLimitNs)) &&
                   __all_sync(kFull, ptx::mbar_wait_bounded(b2, p2, kWaitLimitNs));
        };
        auto issue_s = [&](int j) {
            ptx::tc_fence_after();
            // (columns of blocks past the context come out of stale rows;
            // the causal mask drops them)
            const uint64_t kd = ptx::umma_desc_sw128(kstage(j % kTcKStages), 16,
                                                     tc_group_bytes(D));
            if (ptx::elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    ptx::umma_bf16_ts(s_tm, q_tm + (uint32_t)(kk * 8),
                                      kd + (uint64_t)(((kk >> 2) * 1024 + (kk & 3) * 32) >> 4),
                                      IDESC_S, kk > 0);
                ptx::umma_commit(sfull);
                ptx::umma_commit(kempty + 8u * (j % kTcKStages));
            }
            __syncwarp();
        };
        auto issue_pv = [&](int j) -> bool {
            const int s = j & 1, vs = j % kTcVStages;
            if (!ready(pready + 8u * s, (uint32_t)((j >> 1) & 1), vfull + 8u * vs,
                       (uint32_t)((j / kTcVStages) & 1)))
                return false;
            ptx::tc_fence_after();
            const int nbox = tc_boxes(j, ctx);
            const uint64_t vd = ptx::umma_desc_sw128(vstage(vs), 1024, tc_group_bytes(D));
            if (ptx::elect_one()) {
                for (int box = 0; box < nbox; ++box)
                    ptx::umma_bf16_ts(o_tm, p_tm + (uint32_t)(s * 32 + box * 8),
                                      vd + (uint64_t)((box * BOX) >> 4), IDESC_O,
                                      j > 0 || box > 0);
                ptx::umma_commit(vempty + 8u * vs);
                ptx::umma_commit(pfree + 8u * s);
            }
            __syncwarp();
            return true;
        };
        // One issuing warp, in the order the softmax needs the results: once
        // the softmax has read S_j, first S_{j+1}, then P_{j-1} V_{j-1} (its
        // P was written before S_j was read).  The tensor pipe runs them in
        // that order, so S_{j+1} does not queue behind a P V that only the
        // softmax of tile j + 1 (its P buffer) or a rescale waits for.
        bool ok = true;
        if (warp == 4) {
            ok = ready(qready, 0, kfull, 0);
            if (ok)
                issue_s(0);
            for (int j = 0; ok && j < ntiles; ++j) {
                if (j + 1 < ntiles) {
                    if (!(ok = ready(sfree, (uint32_t)(j & 1),
                                     kfull + 8u * ((j + 1) % kTcKStages),
                                     (uint32_t)(((j + 1) / kTcKStages) & 1))))
                        break;
                    issue_s(j + 1);
                }
                if (j >= 1 && !(ok = issue_pv(j - 1)))
                    break;
            }
            if (ok)
                ok = issue_pv(ntiles - 1);
        }
        if (!ok && lane == 0) {
            report(p.dev_status, PA_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
        }
        __syncwarp();
    } else {
        // ================================================ softmax warps
        const int r = tid;                          // query row = TMEM lane
        // rows past the chunk (not stored) are clamped to the last position
        const int pos = min(pos0 + r / G, ctx - 1);
        const uint32_t lane_tm = (uint32_t)(warp * 32) << 16;
        // with a positive scale the max of the raw logits scales to the max
        // of the scaled ones (rounding is monotone); otherwise scale first
        const bool pos_scale = p.scale_log2 > 0.f;
        const float sc = pos_scale ? p.scale_log2 : 1.f;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = __all_sync(kFull, ptx::mbar_wait_bounded(qfull, 0, kWaitLimitNs));
        // tcgen05.ld / st / wait are .sync.aligned: every decision that
        // guards one is made for the whole warp
        if (ok) {
            // this row of Q, from the swizzled shared copy (column c, 16-byte
            // unit u at c * 16384 + r * 128 + ((u ^ (r & 7)) << 4)) into
            // tensor memory, two bf16 per column
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4) {
                uint32_t w[16];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int u = (c4 & 1) * 4 + k;
                    const uint32_t a = q_s + (uint32_t)((c4 >> 1) * kTcRows * 128 + r * 128) +
                                       ((uint32_t)(u ^ (r & 7)) << 4);
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w[4 * k]), "=r"(w[4 * k + 1]), "=r"(w[4 * k + 2]),
                                   "=r"(w[4 * k + 3])
                                 : "r"(a));
                }
                ptx::tmem_st16(q_tm + lane_tm + (uint32_t)(c4 * 16), w);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            // the Q region is reused by V copies (async proxy)
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(qready);
        }
        for (int j = 0; ok && j < ntiles; ++j) {
            const int s = j & 1;
            // S_j: one non-blocking test; only when it fails, the abort check
            // and the bounded wait
            if (!__all_sync(kFull, ptx::mbar_test_wait(sfull, (uint32_t)(j & 1)))) {
                if (__any_sync(kFull, *abort_flag != 0) ||
                    !__all_sync(kFull, ptx::mbar_wait_bounded(sfull, (uint32_t)(j & 1),
                                                              kWaitLimitNs))) {
                    ok = false;
                    break;
                }
            }
            ptx::tc_fence_after();
            float sv[kTcTile];
            {
                uint32_t u0[16], u1[16], u2[16], u3[16];
                const uint32_t sa = s_tm + lane_tm;
                ptx::tmem_ld16(sa, u0);
                ptx::tmem_ld16(sa + 16, u1);
                ptx::tmem_ld16(sa + 32, u2);
                ptx::tmem_ld16(sa + 48, u3);
                ptx::tmem_wait_ld();
                // S is in registers: the MMA may overwrite it
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    ptx::mbar_arrive(sfree);
                // (the values are taken only after the arrive, so that no
                // arithmetic on them is scheduled ahead of it)
                ptx::tmem_hold16(u0);
                ptx::tmem_hold16(u1);
                ptx::tmem_hold16(u2);
                ptx::tmem_hold16(u3);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    sv[e] = __uint_as_float(u0[e]);
                    sv[16 + e] = __uint_as_float(u1[e]);
                    sv[32 + e] = __uint_as_float(u2[e]);
                    sv[48 + e] = __uint_as_float(u3[e]);
                }
            }
            if (!pos_scale) {
#pragma unroll
                for (int c = 0; c < kTcTile; ++c)
                    sv[c] *= p.scale_log2;
            }
            const int tstart = j * kTcTile;
            if (tstart + kTcTile - 1 > pos0) {
                // a column past some row's position (or past the context)
#pragma unroll
                for (int c = 0; c < kTcTile; ++c)
                    sv[c] = tstart + c <= pos ? sv[c] : -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                m8[e] = sv[e];
#pragma unroll
            for (int c = 8; c < kTcTile; ++c)
                m8[c & 7] = fmaxf(m8[c & 7], sv[c]);
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) *
                             sc;
            bool grow = false;
            float alpha = 1.f;
            if (m_ref == -INFINITY) {
                m_ref = mx;                          // nothing accumulated yet
            } else if (mx > m_ref + 8.f) {
                grow = true;
                alpha = ptx::ex2(m_ref - mx);
            }
            if (__any_sync(kFull, grow)) {
                // O must be stable: P_{j-1} V_{j-1} (and all before) done
                if (!__all_sync(kFull, ptx::mbar_wait_bounded(pfree + 8u * (s ^ 1),
                                                              (uint32_t)(((j - 1) >> 1) & 1),
                                                              kWaitLimitNs))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                // the whole warp rescales its rows of O (alpha = 1 for rows
                // whose max did not grow)
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t u[16];
                    ptx::tmem_ld16(o_tm + lane_tm + (uint32_t)(c * 16), u);
                    ptx::tmem_wait_ld();
                    ptx::tmem_hold16(u);
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
            const float nref = m_ref == -INFINITY ? 0.f : -m_ref;
            // P row as 32 columns of bf16 pairs
            uint32_t w0[16], w1[16];
            float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float e0 = ptx::ex2(fmaf(sv[2 * k], sc, nref));
                const float e1 = ptx::ex2(fmaf(sv[2 * k + 1], sc, nref));
                const float e2 = ptx::ex2(fmaf(sv[32 + 2 * k], sc, nref));
                const float e3 = ptx::ex2(fmaf(sv[32 + 2 * k + 1], sc, nref));
                w0[k] = ptx::pack_bf16x2(e0, e1);
                w1[k] = ptx::pack_bf16x2(e2, e3);
                l4[k & 3] += (e0 + e1) + (e2 + e3);
            }
            l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            if (j >= 2) {
                // P buffer s is free once P_{j-2} V_{j-2} is done (long since,
                // in the usual case: one non-blocking test)
                const uint32_t pph = (uint32_t)(((j - 2) >> 1) & 1);
                if (!__all_sync(kFull, ptx::mbar_test_wait(pfree + 8u * s, pph)) &&
                    !__all_sync(kFull, ptx::mbar_wait_bounded(pfree + 8u * s, pph, kWaitLimitNs))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
            }
            ptx::tmem_st16(p_tm + lane_tm + (uint32_t)(s * 32), w0);
            ptx::tmem_st16(p_tm + lane_tm + (uint32_t)(s * 32 + 16), w1);
            if (tstart + kTcTile > ctx && ((ctx - tstart) & 15) != 0) {
                // V rows of the last block past the context: whatever the
                // pool holds there; their weight is 0, but 0 * NaN is NaN
                if (!__all_sync(kFull, ptx::mbar_wait_bounded(
                                           vfull + 8u * (j % kTcVStages),
                                           (uint32_t)((j / kTcVStages) & 1), kWaitLimitNs))) {
                    ok = false;
                    break;
                }
                const int from = ctx - tstart;
                const int to = (from + 15) & ~15;
                const uint32_t vst = vstage(j % kTcVStages);
                for (int idx = r; idx < (to - from) * NCH * 8; idx += kTcRows) {
                    const int t = from + idx / (NCH * 8), rem = idx % (NCH * 8);
                    const uint32_t a = vst + (uint32_t)((t >> 3) * tc_group_bytes(D) +
                                                        (rem >> 3) * 1024 + (t & 7) * 128 +
                                                        (rem & 7) * 16);
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0)
                                 : "memory");
                }
                // the MMA reads V through the async proxy
                ptx::fence_proxy_async_smem();
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(pready + 8u * s);
        }
        if (ok && !__all_sync(kFull, ptx::mbar_wait_bounded(pfree + 8u * ((ntiles - 1) & 1),
                                                            (uint32_t)(((ntiles - 1) >> 1) & 1),
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
                ptx::tmem_hold16(u);
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
