// Instantiates the decode kernels over an FP8 (E4M3) cache.
#include "pa_launch.cuh"

namespace pa {
pa_status decode_fp8(DecodeLaunch &L, int *grid, bool launch)
{
    return decode_fp8_dispatch(L, grid, launch);
}
}  // namespace pa
