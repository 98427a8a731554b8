// Instantiates the fp32 decode (CUDA-core math) kernels.
#include "pa_launch.cuh"

namespace pa {
pa_status decode_f32(DecodeLaunch &L, int *grid, bool launch)
{
    return decode_dispatch<float, false>(L, grid, launch);
}
}  // namespace pa
