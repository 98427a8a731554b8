// Instantiates the bf16 decode kernels with tensor-core tile math.
#include "pa_launch.cuh"

namespace pa {
pa_status decode_bf16_mma(DecodeLaunch &L, int *grid, bool launch)
{
    return decode_dispatch<__nv_bfloat16, true>(L, grid, launch);
}
}  // namespace pa
