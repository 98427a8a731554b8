// Instantiates the bf16 decode kernels with CUDA-core tile math (kept to
// compare against the tensor-core math on the same data).
#include "pa_launch.cuh"

namespace pa {
pa_status decode_bf16_simt(DecodeLaunch &L, int *grid, bool launch)
{
    return decode_dispatch<__nv_bfloat16, false>(L, grid, launch);
}
}  // namespace pa
