// pa_launch.cuh -- host-side launch templates shared by the translation units
// that instantiate the decode kernels (one per dtype / math).
#pragma once

#include <mutex>

#include "pa_kernels.cuh"

namespace pa {

struct DecodeLaunch {
    DecodeParams p;
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;
    int head_dim;
    int group;
    bool tr16;          // block size >= 16: one 16-row box per tile
    bool kv8;           // the pools hold E4M3 codes (query and output bf16)
    int smem_bytes;
    cudaStream_t stream;
};

// Persistent grid capacity (SMs x resident CTAs) of kernel `fn` with
// `smem_bytes` of dynamic shared memory on the current device; cached.
inline pa_status grid_capacity(const void *fn, int threads, int smem_bytes, int *cap)
{
    struct Slot {
        const void *fn;
        int dev, threads, smem, cap;
    };
    static std::mutex mu;
    static Slot slots[512];
    static int nslots = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PA_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < nslots; ++i)
            if (slots[i].fn == fn && slots[i].dev == dev && slots[i].threads == threads &&
                slots[i].smem == smem_bytes) {
                *cap = slots[i].cap;
                return PA_OK;
            }
    }
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) !=
        cudaSuccess)
        return PA_ERR_CUDA;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return PA_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem_bytes) !=
        cudaSuccess)
        return PA_ERR_CUDA;
    if (per_sm < 1)
        return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (nslots < 512)
        slots[nslots++] = Slot{fn, dev, threads, smem_bytes, sms * per_sm};
    *cap = sms * per_sm;
    return PA_OK;
}

// With launch == false, *grid receives the capacity; otherwise the kernel is
// launched with min(*grid, capacity) CTAs and *grid receives that count.
template <typename T, int D, int G, bool MMA, bool TR16, bool KV8 = false>
pa_status decode_one(DecodeLaunch &L, int *grid, bool launch)
{
    auto fn = &decode_kernel<T, D, G, MMA, TR16, KV8>;
    const int threads = KV8 ? kThreads8 : 32 * (L.p.geo.hpc + 1);
    int cap = 0;
    pa_status st = grid_capacity(reinterpret_cast<const void *>(fn), threads, L.smem_bytes, &cap);
    if (st != PA_OK)
        return st;
    if constexpr (KV8) {
        // the kernel moves registers from its producer warpgroup to its
        // consumers; that needs the launch to hold the registers it assumes
        static int regs = -1;
        if (regs < 0) {
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess)
                return PA_ERR_CUDA;
            regs = fa.numRegs;
        }
        if (regs != kRegsLaunch8)
            return PA_ERR_UNSUPPORTED;
    }
    if (!launch) {
        *grid = cap;
        return PA_OK;
    }
    const int g = *grid < cap ? (*grid > 0 ? *grid : 1) : cap;
    *grid = g;
    // programmatic dependent launch: may start while the previous kernel on
    // the stream runs, if that kernel allows it (the cache write does); the
    // producer waits for it before touching the pools
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)L.smem_bytes;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fn, L.tmap_k, L.tmap_v, L.p) != cudaSuccess)
        return PA_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int D, int G, bool MMA>
pa_status decode_tr(DecodeLaunch &L, int *grid, bool launch)
{
    return L.tr16 ? decode_one<T, D, G, MMA, true>(L, grid, launch)
                  : decode_one<T, D, G, MMA, false>(L, grid, launch);
}

template <typename T, int D, bool MMA>
pa_status decode_g(DecodeLaunch &L, int *grid, bool launch)
{
    switch (L.group) {
    case 1: return decode_tr<T, D, 1, MMA>(L, grid, launch);
    case 2: return decode_tr<T, D, 2, MMA>(L, grid, launch);
    case 4: return decode_tr<T, D, 4, MMA>(L, grid, launch);
    case 8: return decode_tr<T, D, 8, MMA>(L, grid, launch);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T, bool MMA>
pa_status decode_dispatch(DecodeLaunch &L, int *grid, bool launch)
{
    switch (L.head_dim) {
    case 64: return decode_g<T, 64, MMA>(L, grid, launch);
    case 128: return decode_g<T, 128, MMA>(L, grid, launch);
    case 256: return decode_g<T, 256, MMA>(L, grid, launch);
    default: return PA_ERR_UNSUPPORTED;
    }
}

// Entry points of the instantiation units.
pa_status decode_f32(DecodeLaunch &L, int *grid, bool launch);
pa_status decode_fp8(DecodeLaunch &L, int *grid, bool launch);
pa_status decode_bf16_mma(DecodeLaunch &L, int *grid, bool launch);
pa_status decode_bf16_simt(DecodeLaunch &L, int *grid, bool launch);

// Chunked prefill (pa_inst_prefill.cu).
struct PrefillParams;
pa_status prefill_dispatch(int head_dim, int group, const CUtensorMap &tk, const CUtensorMap &tv,
                           const PrefillParams &p, int grid, int smem, cudaStream_t stream);
pa_status prefill_tc_dispatch(int head_dim, int group, const CUtensorMap &tq,
                              const CUtensorMap &tk, const CUtensorMap &tv,
                              const PrefillParams &p, int grid, cudaStream_t stream);

}  // namespace pa
