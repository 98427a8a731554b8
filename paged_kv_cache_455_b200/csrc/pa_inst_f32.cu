// Instantiates the fp32 decode (CUDA-core math) and merge kernels.
#include "pa_launch.cuh"

namespace pa {
pa_status decode_f32(DecodeLaunch &L, int *grid, bool launch)
{
    return decode_dispatch<float, false>(L, grid, launch);
}
pa_status merge_f32(const MergeParams &m, int head_dim, int group, cudaStream_t s)
{
    return merge_dispatch<float>(m, head_dim, group, s);
}
}  // namespace pa
