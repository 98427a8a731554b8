// Instantiates the chunked-prefill kernels (bf16; d = 64, 128, 256; group
// 1, 2, 4, 8) and launches them.
#include <mutex>

#include "pa_prefill.cuh"
#include "pa_prefill_tc.cuh"

namespace pa {
namespace {

template <int D, int G>
pa_status prefill_launch(const CUtensorMap &tk, const CUtensorMap &tv, const PrefillParams &p,
                         int grid, int smem, cudaStream_t stream)
{
    static std::mutex mu;
    static bool ready[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return PA_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!ready[dev]) {
            if (cudaFuncSetAttribute(prefill_kernel<D, G>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemBudget) != cudaSuccess)
                return PA_ERR_CUDA;
            ready[dev] = true;
        }
    }
    prefill_kernel<D, G><<<(unsigned)grid, kPfThreads, smem, stream>>>(tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D>
pa_status prefill_g(int group, const CUtensorMap &tk, const CUtensorMap &tv,
                    const PrefillParams &p, int grid, int smem, cudaStream_t stream)
{
    switch (group) {
    case 1: return prefill_launch<D, 1>(tk, tv, p, grid, smem, stream);
    case 2: return prefill_launch<D, 2>(tk, tv, p, grid, smem, stream);
    case 4: return prefill_launch<D, 4>(tk, tv, p, grid, smem, stream);
    case 8: return prefill_launch<D, 8>(tk, tv, p, grid, smem, stream);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <int D, int G>
pa_status prefill_tc_launch(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const PrefillParams &p, int grid, cudaStream_t stream)
{
    static std::mutex mu;
    static bool ready[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return PA_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!ready[dev]) {
            if (cudaFuncSetAttribute(prefill_tc_kernel<D, G>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemBudget) != cudaSuccess)
                return PA_ERR_CUDA;
            ready[dev] = true;
        }
    }
    prefill_tc_kernel<D, G><<<(unsigned)grid, kTcThreads, tc_smem_bytes(D), stream>>>(tq, tk, tv,
                                                                                    p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D>
pa_status prefill_tc_g(int group, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const PrefillParams &p, int grid,
                       cudaStream_t stream)
{
    switch (group) {
    case 1: return prefill_tc_launch<D, 1>(tq, tk, tv, p, grid, stream);
    case 2: return prefill_tc_launch<D, 2>(tq, tk, tv, p, grid, stream);
    case 4: return prefill_tc_launch<D, 4>(tq, tk, tv, p, grid, stream);
    case 8: return prefill_tc_launch<D, 8>(tq, tk, tv, p, grid, stream);
    default: return PA_ERR_UNSUPPORTED;
    }
}

}  // namespace

pa_status prefill_tc_dispatch(int head_dim, int group, const CUtensorMap &tq,
                              const CUtensorMap &tk, const CUtensorMap &tv,
                              const PrefillParams &p, int grid, cudaStream_t stream)
{
    switch (head_dim) {
    case 64: return prefill_tc_g<64>(group, tq, tk, tv, p, grid, stream);
    case 128: return prefill_tc_g<128>(group, tq, tk, tv, p, grid, stream);
    case 256: return prefill_tc_g<256>(group, tq, tk, tv, p, grid, stream);
    default: return PA_ERR_UNSUPPORTED;
    }
}

pa_status prefill_dispatch(int head_dim, int group, const CUtensorMap &tk, const CUtensorMap &tv,
                           const PrefillParams &p, int grid, int smem, cudaStream_t stream)
{
    switch (head_dim) {
    case 64: return prefill_g<64>(group, tk, tv, p, grid, smem, stream);
    case 128: return prefill_g<128>(group, tk, tv, p, grid, smem, stream);
    case 256: return prefill_g<256>(group, tk, tv, p, grid, smem, stream);
    default: return PA_ERR_UNSUPPORTED;
    }
}

}  // namespace pa
