// Instantiates the decode kernels over an FP8 (E4M3) cache.
#include "pa_launch.cuh"

namespace pa {
// FP8 (E4M3) cache: bf16 query and output, blocks of 16 or 32, d 128 or 256.
template <int D>
pa_status decode_fp8_g(DecodeLaunch &L, int *grid, bool launch)
{
    using B = __nv_bfloat16;
    switch (L.group) {
    case 1: return decode_one<B, D, 1, true, true, true>(L, grid, launch);
    case 2: return decode_one<B, D, 2, true, true, true>(L, grid, launch);
    case 4: return decode_one<B, D, 4, true, true, true>(L, grid, launch);
    case 8: return decode_one<B, D, 8, true, true, true>(L, grid, launch);
    default: return PA_ERR_UNSUPPORTED;
    }
}

inline pa_status decode_fp8_dispatch(DecodeLaunch &L, int *grid, bool launch)
{
    if (!L.tr16)
        return PA_ERR_UNSUPPORTED;
    switch (L.head_dim) {
    case 128: return decode_fp8_g<128>(L, grid, launch);
    case 256: return decode_fp8_g<256>(L, grid, launch);
    default: return PA_ERR_UNSUPPORTED;
    }
}

pa_status decode_fp8(DecodeLaunch &L, int *grid, bool launch)
{
    return decode_fp8_dispatch(L, grid, launch);
}
}  // namespace pa
