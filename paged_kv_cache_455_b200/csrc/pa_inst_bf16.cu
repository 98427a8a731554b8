// Instantiates the bf16 decode kernels with tensor-core tile math, and the
// bf16 merge kernels.
#include "pa_launch.cuh"

namespace pa {
pa_status decode_bf16_mma(DecodeLaunch &L, int *grid, bool launch)
{
    return decode_dispatch<__nv_bfloat16, true>(L, grid, launch);
}
pa_status merge_bf16(const MergeParams &m, int head_dim, int group, cudaStream_t s)
{
    return merge_dispatch<__nv_bfloat16>(m, head_dim, group, s);
}
}  // namespace pa
