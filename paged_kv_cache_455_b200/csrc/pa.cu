// pa.cu -- C ABI of the paged KV-cache decode library: argument checks,
// shared-memory geometry, TMA tensor maps, work-decomposition choice and
// launches.  Device code lives in pa_kernels.cuh; the decode kernels
// are instantiated in pa_inst_*.cu.
//
// pa_decode_attention uses the stream-K decomposition (mode 0) when the
// caller's workspace holds the partial states of the cut segments, and whole
// segments per CTA (mode 1) otherwise.  pa_decode_splitk runs mode 1 over
// fixed partitions.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cmath>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "pa.h"
#include "pa_testing.h"
#include "pa_launch.cuh"
#include "pa_prefill.cuh"

namespace {

using pa::DecodeLaunch;
using pa::DecodeParams;
using pa::TileGeo;

std::atomic<unsigned long long> g_launches{0};

// Test hooks (include/pa_testing.h): the bounded-wait limit of the decode
// kernels and a CTA whose producer withholds one tile's copies.
std::atomic<unsigned long long> g_test_wait_ns{0};
std::atomic<int> g_test_withhold{-1};

// Bound on decode CTAs used to size the stream-K workspace (one per SM, up
// to 256 SMs).
constexpr int kWorkspaceCtas = 256;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ilog2_exact(int v)
{
    int s = 0;
    while ((1 << s) < v)
        ++s;
    return (1 << s) == v ? s : -1;
}

int64_t round_up(int64_t v, int64_t m) { return ((v + m - 1) / m) * m; }

int elem_size(pa_dtype dt) { return dt == PA_DTYPE_F32 ? 4 : (dt == PA_DTYPE_FP8_E4M3 ? 1 : 2); }

// =====================================================================
// Cache write kernel: one warp per (token, KV head, K|V) row, 16-byte copies.
// =====================================================================
struct CacheParams {
    const void *key;
    const void *value;
    void *k_pool;
    void *v_pool;
    const int64_t *slot_mapping;
    int32_t *dev_status;
    int64_t num_slots;      // nb * bs
    int num_tokens;
    int num_kv_heads;
    int row_bytes;          // d * element size
};

__global__ void __launch_bounds__(256) cache_write_kernel(const CacheParams p)
{
    // the decode kernel that follows may start its set-up now; it waits for
    // this grid to finish before reading the pools
    pa::ptx::grid_launch_dependents();
    // launched as a programmatic dependent of the kernel ahead: its inputs
    // (and readers of the pools) must be done before anything is touched
    pa::ptx::grid_wait_prerequisites();
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nrows = (int64_t)p.num_tokens * p.num_kv_heads * 2;
    if (row >= nrows)
        return;
    const int kv = (int)(row & 1);
    const int64_t th = row >> 1;
    const int64_t t = th / p.num_kv_heads;
    const int64_t h = th - t * p.num_kv_heads;
    const int64_t slot = p.slot_mapping[t];
    if (slot < 0)
        return;
    if (slot >= p.num_slots) {
        if (lane == 0 && h == 0 && kv == 0)
            pa::report(p.dev_status, PA_DEV_BAD_SLOT);
        return;
    }
    const int4 *src = reinterpret_cast<const int4 *>(
        static_cast<const uint8_t *>(kv ? p.value : p.key) + (t * p.num_kv_heads + h) * p.row_bytes);
    int4 *dst = reinterpret_cast<int4 *>(static_cast<uint8_t *>(kv ? p.v_pool : p.k_pool) +
                                         (slot * p.num_kv_heads + h) * p.row_bytes);
    const int n16 = p.row_bytes >> 4;
    for (int c = lane; c < n16; c += 32)
        dst[c] = __ldg(src + c);
}

struct CacheFp8Params {
    const __nv_bfloat16 *key;
    const __nv_bfloat16 *value;
    uint8_t *k_pool;
    uint8_t *v_pool;
    const int64_t *slot_mapping;
    int32_t *dev_status;
    int64_t num_slots;      // nb * bs
    int num_tokens;
    int num_kv_heads;
    int head_dim;
    float k_scale;
    float v_scale;
};

// Cache write into E4M3 pools: one warp per (token, KV head, K|V) row; a
// lane turns 8 bf16 elements into the E4M3 codes of element / scale (the
// division rounded as binary32, then to nearest E4M3, ties to even,
// saturating at +-448) and stores them as one 8-byte word.
__global__ void __launch_bounds__(256) cache_write_fp8_kernel(const CacheFp8Params p)
{
    pa::ptx::grid_launch_dependents();
    pa::ptx::grid_wait_prerequisites();
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nrows = (int64_t)p.num_tokens * p.num_kv_heads * 2;
    if (row >= nrows)
        return;
    const int kv = (int)(row & 1);
    const int64_t th = row >> 1;
    const int64_t t = th / p.num_kv_heads;
    const int64_t h = th - t * p.num_kv_heads;
    const int64_t slot = p.slot_mapping[t];
    if (slot < 0)
        return;
    if (slot >= p.num_slots) {
        if (lane == 0 && h == 0 && kv == 0)
            pa::report(p.dev_status, PA_DEV_BAD_SLOT);
        return;
    }
    const float sc = kv ? p.v_scale : p.k_scale;
    const uint4 *src = reinterpret_cast<const uint4 *>((kv ? p.value : p.key) +
                                                       (t * p.num_kv_heads + h) * p.head_dim);
    uint2 *dst = reinterpret_cast<uint2 *>((kv ? p.v_pool : p.k_pool) +
                                           (slot * p.num_kv_heads + h) * p.head_dim);
    for (int c = lane; c < (p.head_dim >> 3); c += 32) {
        const uint4 in = __ldg(src + c);
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
        uint32_t packed[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint32_t v = 0;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t b = w[2 * i + j];
                const float x0 = __fdiv_rn(pa::ptx::bf16lo_to_f32(b), sc);
                const float x1 = __fdiv_rn(pa::ptx::bf16hi_to_f32(b), sc);
                const uint32_t two = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(x0, x1),
                                                                        __NV_SATFINITE, __NV_E4M3);
                v |= (two & 0xffffu) << (16 * j);
            }
            packed[i] = v;
        }
        dst[c] = make_uint2(packed[0], packed[1]);
    }
}

struct CopyParams {
    const void *src_k;
    const void *src_v;
    void *dst_k;
    void *dst_v;
    const int64_t *block_mapping;   // [num_pairs][2]: source, destination
    int32_t *dev_status;
    int64_t src_blocks;
    int64_t dst_blocks;
    int64_t block_bytes;            // bs * Hkv * d * element size
    int num_pairs;
};

// One CTA per (pair, pool, 8 KB chunk of the block): 16-byte copies, 512
// bytes per warp instruction.  Either side may be pinned host memory mapped
// into the device's address space (swap).
__global__ void __launch_bounds__(256) copy_blocks_kernel(const CopyParams p, int chunks)
{
    const int pair = blockIdx.x / (2 * chunks);
    const int rest = blockIdx.x - pair * 2 * chunks;
    const int kv = rest / chunks;
    const int chunk = rest - kv * chunks;
    const int64_t src = p.block_mapping[2 * pair];
    const int64_t dst = p.block_mapping[2 * pair + 1];
    if (src < 0 || src >= p.src_blocks || dst < 0 || dst >= p.dst_blocks) {
        if (threadIdx.x == 0 && kv == 0 && chunk == 0)
            pa::report(p.dev_status, PA_DEV_BAD_BLOCK);
        return;
    }
    const int4 *from = reinterpret_cast<const int4 *>(
        static_cast<const uint8_t *>(kv ? p.src_v : p.src_k) + src * p.block_bytes);
    int4 *to = reinterpret_cast<int4 *>(static_cast<uint8_t *>(kv ? p.dst_v : p.dst_k) +
                                        dst * p.block_bytes);
    const int64_t n16 = p.block_bytes >> 4;
    const int64_t end = min(n16, (int64_t)(chunk + 1) * 512);
    for (int64_t c = (int64_t)chunk * 512 + threadIdx.x; c < end; c += 256)
        to[c] = __ldcg(from + c);
}

// True if the GPU can read and write `ptr` at that same address: device
// memory, or pinned host memory mapped into the unified address space.
bool device_addressable(const void *ptr)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        cudaGetLastError();   // clear the error of an unknown pointer
        return false;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged)
        return true;
    return a.type == cudaMemoryTypeHost && a.devicePointer == ptr;
}

pa_status launch_copy(CopyParams &p, int block_size, int num_kv_heads, int head_dim,
                      pa_dtype dtype, void *stream)
{
    if (p.num_pairs < 0 || p.src_blocks <= 0 || p.dst_blocks <= 0 || num_kv_heads <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16 && dtype != PA_DTYPE_FP8_E4M3)
        return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return PA_ERR_UNSUPPORTED;
    if (ilog2_exact(block_size) < 0 || block_size < 4 || block_size > 32)
        return PA_ERR_UNSUPPORTED;
    if (p.num_pairs == 0)
        return PA_OK;
    if (!p.src_k || !p.src_v || !p.dst_k || !p.dst_v || !p.block_mapping)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(p.src_k) || !aligned16(p.src_v) || !aligned16(p.dst_k) || !aligned16(p.dst_v))
        return PA_ERR_INVALID_ARG;
    if (!device_addressable(p.src_k) || !device_addressable(p.src_v) ||
        !device_addressable(p.dst_k) || !device_addressable(p.dst_v) ||
        !device_addressable(p.block_mapping))
        return PA_ERR_INVALID_ARG;   // e.g. pageable host memory
    p.block_bytes = (int64_t)block_size * num_kv_heads * head_dim * elem_size(dtype);
    const int chunks = (int)((p.block_bytes + 8191) / 8192);
    const int64_t blocks = (int64_t)p.num_pairs * 2 * chunks;
    if (blocks > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    copy_blocks_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(p, chunks);
    ++g_launches;
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// =====================================================================
// Tensor maps
// =====================================================================
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

struct MapKey {
    const void *base;
    int64_t rows;
    int hkv, d, es, tr, hpc, cpb;
    bool operator==(const MapKey &o) const
    {
        return base == o.base && rows == o.rows && hkv == o.hkv && d == o.d && es == o.es &&
               tr == o.tr && hpc == o.hpc && cpb == o.cpb;
    }
};

struct MapEntry {
    MapKey key;
    alignas(64) CUtensorMap map;
};

std::mutex g_map_mu;
MapEntry g_maps[128];
int g_nmaps = 0, g_next_map = 0;

// Tensor map over a pool [nb, bs, Hkv, d] with dims (elements of a 128-byte
// column, token row, column, head) -- the row stride precedes the column
// stride, so a box lands in shared memory as [head][column][row] -- and a box
// of `tr` token rows x d of `hpc` heads, 128-byte swizzled.
// Box: `tr` rows of `hpc` heads, landing in shared memory as
// [head][128-byte column][row][128 bytes].  With `grouped`, the rows are
// split into groups of 8 (a fifth dimension) and a box of `tr` rows of one
// head lands as [8-row group][column][row][128 bytes], so that 8-row groups
// are a fixed stride apart whatever the number of columns.
bool encode_pool_map(CUtensorMap *out, const void *base, int64_t nb, int bs, int hkv, int d,
                     pa_dtype dt, int tr, int hpc, bool grouped = false)
{
    const int es = elem_size(dt);
    const MapKey key{base, nb * bs, hkv, d, es, tr, hpc, grouped ? 1 : 0};
    {
        std::lock_guard<std::mutex> lock(g_map_mu);
        for (int i = 0; i < g_nmaps; ++i)
            if (g_maps[i].key == key) {
                *out = g_maps[i].map;
                return true;
            }
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    const CUtensorMapDataType type =
        dt == PA_DTYPE_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                           : (dt == PA_DTYPE_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    const cuuint32_t epc = 128 / es;           // elements per 128-byte column
    const cuuint64_t rowb = (cuuint64_t)d * es;
    const cuuint32_t nch = (cuuint32_t)(rowb / 128);
    alignas(64) CUtensorMap map;
    CUresult r;
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if (!grouped) {
        const cuuint64_t dims[4] = {epc, (cuuint64_t)(nb * bs), nch, (cuuint64_t)hkv};
        const cuuint64_t strides[3] = {(cuuint64_t)hkv * rowb, 128, rowb};
        const cuuint32_t box[4] = {epc, (cuuint32_t)tr, nch, (cuuint32_t)hpc};
        r = enc(&map, type, 4, const_cast<void *>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        if (bs % 8 != 0 || tr % 8 != 0 || hpc != 1)
            return false;
        const cuuint64_t dims[5] = {epc, 8, nch, (cuuint64_t)(nb * bs / 8), (cuuint64_t)hkv};
        const cuuint64_t strides[4] = {(cuuint64_t)hkv * rowb, 128, 8 * (cuuint64_t)hkv * rowb,
                                       rowb};
        const cuuint32_t box[5] = {epc, 8, nch, (cuuint32_t)(tr / 8), 1};
        r = enc(&map, type, 5, const_cast<void *>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS)
        return false;
    *out = map;
    std::lock_guard<std::mutex> lock(g_map_mu);
    const int slot = g_nmaps < 128 ? g_nmaps++ : (g_next_map++ % 128);
    g_maps[slot].key = key;
    g_maps[slot].map = map;
    return true;
}

// =====================================================================
// Geometry and launch plumbing
// =====================================================================
// KV heads per CTA tile: the largest of 4, 2, 1 dividing Hkv.
int heads_per_cta(int hkv) { return hkv % 4 == 0 ? 4 : (hkv % 2 == 0 ? 2 : 1); }

bool make_geo(TileGeo &g, int D, int es, int es_q, int bs, int group, int hpc, int *smem)
{
    const int rowb = D * es;
    const int nch = rowb / 128;
    g.tr = std::min(16, bs);
    g.tr_log2 = ilog2_exact(g.tr);
    g.bpt = 16 / g.tr;
    g.hpc = hpc;
    g.head_lines = nch * g.tr;
    g.box_stride = (int)round_up((int64_t)hpc * g.head_lines * 128, 1024);
    g.kv_bytes = g.bpt * g.box_stride;
    // over an E4M3 cache a stage holds two consecutive tiles of a segment
    // (64 KB at d = 256, as one bf16 tile)
    g.tps = es == 1 ? 2 : 1;
    g.q_head_bytes = group * D * es_q;
    // an E4M3 cache's stages carry no query rows (its consumer warps read
    // them from global memory)
    g.q_bytes = es == 1 ? 0 : hpc * g.q_head_bytes;
    g.q_off = 2 * g.tps * g.kv_bytes;
    g.stage_bytes = (int)round_up((int64_t)g.q_off + g.q_bytes, 1024);
    g.box_tx = hpc * g.tr * rowb;
    const int fixed = pa::decode_smem_fixed(group, D, es == 1);   // es 1: an E4M3 cache
    const int spw =
        std::min(es == 1 ? pa::kMaxSpw : pa::kMaxSpw16, (pa::kSmemBudget - fixed) / g.stage_bytes);
    if (spw < 1)
        return false;
    g.spw = spw;
    *smem = fixed + spw * g.stage_bytes;
    return true;
}

// bf16 uses the tensor-core tile math unless PA_DECODE_MATH=simt is set
// (kept to compare the two on the same data).
bool bf16_use_mma()
{
    const char *v = std::getenv("PA_DECODE_MATH");
    return !(v && std::strcmp(v, "simt") == 0);
}

pa_status decode_call(DecodeLaunch &L, pa_dtype dtype, int *grid, bool launch)
{
    if (L.kv8)
        return pa::decode_fp8(L, grid, launch);
    if (dtype == PA_DTYPE_F32)
        return pa::decode_f32(L, grid, launch);
    if (bf16_use_mma())
        return pa::decode_bf16_mma(L, grid, launch);
    return pa::decode_bf16_simt(L, grid, launch);
}

pa_status check_attention_args(const void *out, const void *query, const void *k_pool,
                               const void *v_pool, const int32_t *block_tables, int max_blocks,
                               const int32_t *context_lens, int num_seqs, int max_context_len,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int64_t num_blocks, pa_dtype dtype, int *group_out,
                               int *bs_log2_out)
{
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks <= 0 || max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16)
        return PA_ERR_UNSUPPORTED;
    const int group = num_q_heads / num_kv_heads;
    if (group != 1 && group != 2 && group != 4 && group != 8)
        return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return PA_ERR_UNSUPPORTED;
    const int bs_log2 = ilog2_exact(block_size);
    if (block_size < 4 || block_size > 32 || bs_log2 < 0)
        return PA_ERR_UNSUPPORTED;
    if ((int64_t)max_context_len > (int64_t)max_blocks * block_size)
        return PA_ERR_INVALID_ARG;
    if (num_blocks > (int64_t)INT32_MAX / block_size)
        return PA_ERR_INVALID_ARG;   // token rows of the pool are int32 TMA coordinates
    if ((int64_t)num_kv_heads > 256)
        return PA_ERR_UNSUPPORTED;   // TMA tensor dims
    // every tile index of the batch must fit an int
    if ((int64_t)num_seqs * num_kv_heads * (round_up((int64_t)max_blocks * block_size, 16) / 16) >
        (int64_t)INT32_MAX / 2)
        return PA_ERR_INVALID_ARG;
    if (num_seqs > 0) {
        if (!out || !query || !k_pool || !v_pool || !block_tables || !context_lens)
            return PA_ERR_INVALID_ARG;
        if (!aligned16(out) || !aligned16(query) || !aligned16(k_pool) || !aligned16(v_pool))
            return PA_ERR_INVALID_ARG;
    }
    *group_out = group;
    *bs_log2_out = bs_log2;
    return PA_OK;
}

// Fills everything of a decode launch but the work decomposition.
pa_status prepare_decode(DecodeLaunch &L, void *out, const void *query, const void *k_pool,
                         const void *v_pool, const int32_t *block_tables, int max_blocks,
                         const int32_t *context_lens, int num_seqs, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int bs_log2,
                         int64_t num_blocks, float scale, pa_dtype dtype, int group,
                         int32_t *dev_status, void *stream, bool kv8 = false,
                         float k_scale = 1.f, float v_scale = 1.f)
{
    std::memset(&L.p, 0, sizeof(L.p));
    DecodeParams &p = L.p;
    p.out = out;
    p.q = query;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.dev_status = dev_status;
    p.num_blocks = num_blocks;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.max_blocks = max_blocks;
    p.block_size = block_size;
    p.bs_log2 = bs_log2;
    // an FP8 cache's K scale multiplies every logit, its V scale every output
    p.scale_log2 = kv8 ? scale * k_scale * pa::kLog2e : scale * pa::kLog2e;
    p.out_scale = kv8 ? v_scale : 1.f;
    const unsigned long long wait_ns = g_test_wait_ns.load();
    p.wait_ns = wait_ns ? wait_ns : pa::kWaitLimitNs;
    p.withhold_cta = g_test_withhold.load();
    L.head_dim = head_dim;
    L.group = group;
    L.tr16 = block_size >= 16;
    L.kv8 = kv8;
    L.stream = static_cast<cudaStream_t>(stream);
    const pa_dtype pool_dtype = kv8 ? PA_DTYPE_FP8_E4M3 : dtype;
    const int es = elem_size(pool_dtype);
    const int tr = std::min(16, block_size);
    const int hpc = heads_per_cta(num_kv_heads);
    p.head_groups = num_kv_heads / hpc;
    if (!make_geo(p.geo, head_dim, es, elem_size(dtype), block_size, group, hpc, &L.smem_bytes))
        return PA_ERR_UNSUPPORTED;
    if (!encode_pool_map(&L.tmap_k, k_pool, num_blocks, block_size, num_kv_heads, head_dim,
                         pool_dtype, tr, hpc) ||
        !encode_pool_map(&L.tmap_v, v_pool, num_blocks, block_size, num_kv_heads, head_dim,
                         pool_dtype, tr, hpc))
        return PA_ERR_CUDA;
    return PA_OK;
}

// Floats of one partial slot: the accumulator (G*D floats, the tensor-core
// layout padding an odd group to an even one), max [G], sum [G], bad mark.
int64_t slot_floats(int64_t group, int64_t head_dim)
{
    return round_up(pa::piece_stats_off((int)head_dim, (int)group) + 2 * group + 1, 4);
}

// Stream-K workspace: two partial slots per CTA and head of the group (a CTA
// holds at most two pieces of cut segments: one met at the start of its
// range, one running past its end); from the next 128-byte boundary, one
// arrival counter per CTA and head (for the cut segment that starts in the
// CTA's range), each on a 128-byte line of its own.
int64_t partials_bytes(int64_t heads, int64_t group, int64_t head_dim)
{
    return round_up(2 * heads * slot_floats(group, head_dim) * 4, 128);
}

size_t stream_k_bytes(int64_t num_seqs, int64_t num_kv_heads, int64_t group, int64_t head_dim,
                      int64_t ctas)
{
    (void)num_seqs;
    const int64_t heads = ctas * heads_per_cta((int)num_kv_heads);
    return (size_t)(partials_bytes(heads, group, head_dim) + heads * 128);
}

// Epoch of a stream-K call: the tag its arrival counters carry.  Distinct
// for consecutive calls of this process and never 0; the sequence starts at
// a clock-derived value, so counters another process left in reused device
// memory are unlikely (about 2^-32 per counter) to match.
uint32_t epoch_seed()
{
    uint64_t x = (uint64_t)std::chrono::high_resolution_clock::now().time_since_epoch().count();
    x ^= x >> 33;
    x *= 0xff51afd7ed558ccdull;
    x ^= x >> 33;
    return (uint32_t)x;
}

uint32_t next_epoch()
{
    static std::atomic<uint32_t> counter{epoch_seed()};
    uint32_t e;
    do {
        e = ++counter;
    } while (e == 0);
    return e;
}

pa_status launch_reduce(void *out, const float *tmp_out, const float *max_logits,
                        const float *exp_sums, const int32_t *context_lens, int num_seqs,
                        int num_q_heads, int head_dim, int partition_size, int max_parts,
                        int ctx_cap, pa_dtype dtype, cudaStream_t stream)
{
    pa::ReduceParams rp;
    rp.out = out;
    rp.tmp_out = tmp_out;
    rp.max_logits = max_logits;
    rp.exp_sums = exp_sums;
    rp.context_lens = context_lens;
    rp.num_seqs = num_seqs;
    rp.num_q_heads = num_q_heads;
    rp.partition_size = partition_size;
    rp.max_parts = max_parts;
    rp.ctx_cap = ctx_cap;
    const int64_t grid = (int64_t)num_seqs * num_q_heads;
    if (grid > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    if (dtype == PA_DTYPE_F32)
        pa::reduce_kernel<float><<<(unsigned)grid, 128, 0, stream>>>(rp, head_dim);
    else
        pa::reduce_kernel<__nv_bfloat16><<<(unsigned)grid, 128, 0, stream>>>(rp, head_dim);
    ++g_launches;
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t splitk_bytes(int64_t num_seqs, int64_t num_q_heads, int64_t head_dim, int64_t parts)
{
    return (size_t)(num_seqs * num_q_heads * parts * (head_dim + 2) * 4);
}

// =====================================================================
// Scratch for pa_decode_attention_static: a fixed array in device memory,
// allocated when the library is loaded on a device and held until exit.
// Host code must not pass `g_static_scratch` to a kernel (on the host the
// name is only a stand-in for the symbol); its device address comes from
// cudaGetSymbolAddress, looked up once per device below.
// =====================================================================
static __device__ __align__(256) unsigned char g_static_scratch[PA_STATIC_SCRATCH_BYTES];

std::mutex g_static_mu;
void *g_static_addr[64] = {};

// Device address of g_static_scratch on the current device (nullptr on error).
void *static_scratch_address()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_addr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess)
            return nullptr;
        g_static_addr[dev] = ptr;
    }
    return g_static_addr[dev];
}

// Scratch bytes pa_decode_attention needs for its split over the current
// device's grid (0 when these sizes run without one).
pa_status stream_k_need(size_t *need, const void *out, const void *query, const void *k_pool,
                        const void *v_pool, const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *context_lens, int num_seqs, int max_context_len,
                        int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                        int64_t num_blocks, float scale, pa_dtype dtype)
{
    int group = 0, bs_log2 = 0;
    pa_status st = check_attention_args(out, query, k_pool, v_pool, block_tables,
                                        max_blocks_per_seq, context_lens, num_seqs,
                                        max_context_len, num_q_heads, num_kv_heads, head_dim,
                                        block_size, num_blocks, dtype, &group, &bs_log2);
    if (st != PA_OK)
        return st;
    *need = 0;
    if (num_seqs == 0)
        return PA_OK;
    DecodeLaunch L;
    st = prepare_decode(L, const_cast<void *>(out), query, k_pool, v_pool, block_tables,
                        max_blocks_per_seq, context_lens, num_seqs, num_q_heads, num_kv_heads,
                        head_dim, block_size, bs_log2, num_blocks, scale, dtype, group, nullptr,
                        nullptr);
    if (st != PA_OK)
        return st;
    int grid = 0;
    st = decode_call(L, dtype, &grid, false);
    if (st != PA_OK)
        return st;
    const int64_t tiles_up = (int64_t)num_seqs * L.p.head_groups *
                             (round_up(std::max(max_context_len, 1), 16) / 16);
    grid = (int)std::min<int64_t>(grid, tiles_up);
    *need = stream_k_bytes(num_seqs, num_kv_heads, group, head_dim, grid);
    return PA_OK;
}

}  // namespace

extern "C" {

const char *pa_status_string(pa_status status)
{
    switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported head_dim, block_size, group or dtype";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
    }
}

unsigned long long pa_launch_count(void) { return g_launches.load(); }

void pa_testing_set_wait_limit_ns(unsigned long long ns) { g_test_wait_ns.store(ns); }

void pa_testing_withhold_copy(int cta) { g_test_withhold.store(cta < 0 ? -1 : cta); }

int pa_num_partitions(int max_context_len, int partition_size)
{
    if (partition_size <= 0 || max_context_len <= 0)
        return 1;
    return (int)(((int64_t)max_context_len + partition_size - 1) / partition_size);
}

size_t pa_splitk_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_partitions)
{
    if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_partitions <= 0)
        return 0;
    return splitk_bytes(num_seqs, num_q_heads, head_dim, max_partitions);
}

size_t pa_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_context_len)
{
    (void)max_context_len;
    if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        num_q_heads % num_kv_heads != 0)
        return 0;
    return stream_k_bytes(num_seqs, num_kv_heads, num_q_heads / num_kv_heads, head_dim,
                          kWorkspaceCtas);
}

pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_pool, void *v_pool,
                               const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                               int32_t *dev_status, void *stream)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16)
        return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return PA_ERR_UNSUPPORTED;
    if (ilog2_exact(block_size) < 0 || block_size < 4 || block_size > 32)
        return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0)
        return PA_OK;
    if (!key || !value || !k_pool || !v_pool || !slot_mapping)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_pool) || !aligned16(v_pool))
        return PA_ERR_INVALID_ARG;
    CacheParams p;
    p.key = key;
    p.value = value;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.slot_mapping = slot_mapping;
    p.dev_status = dev_status;
    p.num_slots = num_blocks * block_size;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.row_bytes = head_dim * elem_size(dtype);
    const int64_t rows = (int64_t)num_tokens * num_kv_heads * 2;
    const int64_t blocks = (rows + 7) / 8;   // 8 warps per CTA
    if (blocks > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    // a programmatic dependent of the kernel ahead (its CTAs may be placed on
    // SMs that kernel has left, and wait there for it to complete)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, cache_write_kernel, p);
    ++g_launches;
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_pool, void *v_pool,
                                   const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                                   int head_dim, int block_size, int64_t num_blocks,
                                   float k_scale, float v_scale, int32_t *dev_status, void *stream)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
        return PA_ERR_INVALID_ARG;
    if ((head_dim != 128 && head_dim != 256) || (block_size != 16 && block_size != 32))
        return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0)
        return PA_OK;
    if (!key || !value || !k_pool || !v_pool || !slot_mapping)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_pool) || !aligned16(v_pool))
        return PA_ERR_INVALID_ARG;
    CacheFp8Params p;
    p.key = static_cast<const __nv_bfloat16 *>(key);
    p.value = static_cast<const __nv_bfloat16 *>(value);
    p.k_pool = static_cast<uint8_t *>(k_pool);
    p.v_pool = static_cast<uint8_t *>(v_pool);
    p.slot_mapping = slot_mapping;
    p.dev_status = dev_status;
    p.num_slots = num_blocks * block_size;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    const int64_t rows = (int64_t)num_tokens * num_kv_heads * 2;
    const int64_t blocks = (rows + 7) / 8;   // 8 warps per CTA
    if (blocks > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, cache_write_fp8_kernel, p);
    ++g_launches;
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(void *k_pool, void *v_pool, const int64_t *block_mapping, int num_pairs,
                         int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                         pa_dtype dtype, int32_t *dev_status, void *stream)
{
    CopyParams p;
    p.src_k = k_pool;
    p.src_v = v_pool;
    p.dst_k = k_pool;
    p.dst_v = v_pool;
    p.block_mapping = block_mapping;
    p.dev_status = dev_status;
    p.src_blocks = num_blocks;
    p.dst_blocks = num_blocks;
    p.num_pairs = num_pairs;
    return launch_copy(p, block_size, num_kv_heads, head_dim, dtype, stream);
}

pa_status pa_swap_blocks(void *dst_k_pool, void *dst_v_pool, int64_t dst_num_blocks,
                         const void *src_k_pool, const void *src_v_pool, int64_t src_num_blocks,
                         const int64_t *block_mapping, int num_pairs, int block_size,
                         int num_kv_heads, int head_dim, pa_dtype dtype, int32_t *dev_status,
                         void *stream)
{
    CopyParams p;
    p.src_k = src_k_pool;
    p.src_v = src_v_pool;
    p.dst_k = dst_k_pool;
    p.dst_v = dst_v_pool;
    p.block_mapping = block_mapping;
    p.dev_status = dev_status;
    p.src_blocks = src_num_blocks;
    p.dst_blocks = dst_num_blocks;
    p.num_pairs = num_pairs;
    return launch_copy(p, block_size, num_kv_heads, head_dim, dtype, stream);
}

pa_status pa_prefill_attention(void *out, const void *query, const int32_t *cu_q_lens, int total_q,
                               int max_q_len, const void *k_pool, const void *v_pool,
                               const int32_t *block_tables, int max_blocks_per_seq,
                               const int32_t *context_lens, int num_seqs, int max_context_len,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int64_t num_blocks, float scale, pa_dtype dtype,
                               int32_t *dev_status, void *stream)
{
    if (num_seqs < 0 || total_q < 0 || max_q_len < 0 || max_context_len < 0 ||
        num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
        num_q_heads % num_kv_heads != 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_BF16)
        return PA_ERR_UNSUPPORTED;
    const int group = num_q_heads / num_kv_heads;
    const int bs_log2 = ilog2_exact(block_size);
    if ((head_dim != 64 && head_dim != 128 && head_dim != 256) || bs_log2 < 2 || bs_log2 > 5 ||
        (group != 1 && group != 2 && group != 4 && group != 8))
        return PA_ERR_UNSUPPORTED;
    if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * block_size ||
        max_q_len > std::max(max_context_len, 0))
        return PA_ERR_INVALID_ARG;
    if ((int64_t)max_context_len > (int64_t)pa::kPfMaxBlocks * block_size)
        return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0 || total_q == 0 || max_q_len == 0)
        return PA_OK;
    if (!out || !query || !cu_q_lens || !k_pool || !v_pool || !block_tables || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(query) || !aligned16(k_pool) || !aligned16(v_pool))
        return PA_ERR_INVALID_ARG;
    pa::PrefillParams p;
    p.out = out;
    p.q = query;
    p.cu_q_lens = cu_q_lens;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.dev_status = dev_status;
    p.num_blocks = num_blocks;
    p.total_q = total_q;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.max_blocks = max_blocks_per_seq;
    p.block_size = block_size;
    p.bs_log2 = bs_log2;
    p.tr = std::min(16, block_size);
    p.tr_log2 = ilog2_exact(p.tr);
    p.ctx_cap = std::min(max_blocks_per_seq, pa::kPfMaxBlocks) * block_size;
    const int tq = pa::kPfRows / group;
    p.qblocks = (max_q_len + tq - 1) / tq;
    p.box_stride = pa::prefill_box_stride(p.tr, head_dim);
    const int stage = pa::prefill_stage_bytes(p.tr, head_dim);
    const int fixed = pa::prefill_fixed_bytes(head_dim);
    p.stages = std::min(pa::kPfMaxStages, (pa::kSmemBudget - fixed) / stage);
    if (p.stages < 2)
        return PA_ERR_UNSUPPORTED;
    p.scale_log2 = scale * 1.4426950408889634f;
    const int smem = fixed + p.stages * stage;
    const int64_t grid = (int64_t)num_seqs * num_kv_heads * p.qblocks;
    if (grid > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    // the tensor-core kernel takes 16-row boxes as [8-row group][column][row]
    const bool grouped = block_size >= 16;
    CUtensorMap tk, tv;
    if (!encode_pool_map(&tk, k_pool, num_blocks, block_size, num_kv_heads, head_dim, dtype, p.tr,
                         1, grouped) ||
        !encode_pool_map(&tv, v_pool, num_blocks, block_size, num_kv_heads, head_dim, dtype, p.tr,
                         1, grouped))
        return PA_ERR_CUDA;
    pa_status st;
    if (block_size >= 16) {
        // 5th-generation tensor cores: the query rows of the CTA come by TMA
        // through a 3-D map over [total_q, Hq, d] (box: 64 elements, the
        // group's heads, the CTA's tokens)
        EncodeTiledFn enc = encode_fn();
        if (!enc)
            return PA_ERR_CUDA;
        alignas(64) CUtensorMap qmap;
        const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads,
                                    (cuuint64_t)total_q};
        const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2,
                                       (cuuint64_t)num_q_heads * head_dim * 2};
        const cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)tq};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(query), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return PA_ERR_CUDA;
        st = pa::prefill_tc_dispatch(head_dim, group, qmap, tk, tv, p, (int)grid,
                                     static_cast<cudaStream_t>(stream));
    } else {
        st = pa::prefill_dispatch(head_dim, group, tk, tv, p, (int)grid, smem,
                                  static_cast<cudaStream_t>(stream));
    }
    ++g_launches;
    return st;
}

pa_status pa_decode_splitk(void *out, const void *query, const void *k_pool, const void *v_pool,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int num_seqs, int max_context_len,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int64_t num_blocks, float scale, pa_dtype dtype, int partition_size,
                           int max_partitions, float *tmp_out, float *max_logits,
                           float *exp_sums, int32_t *dev_status, void *stream)
{
    int group = 0, bs_log2 = 0;
    pa_status st = check_attention_args(out, query, k_pool, v_pool, block_tables,
                                        max_blocks_per_seq, context_lens, num_seqs,
                                        max_context_len, num_q_heads, num_kv_heads, head_dim,
                                        block_size, num_blocks, dtype, &group, &bs_log2);
    if (st != PA_OK)
        return st;
    if (partition_size <= 0 || partition_size % pa::kTile != 0 || max_partitions <= 0)
        return PA_ERR_INVALID_ARG;
    if (max_partitions < pa_num_partitions(max_context_len, partition_size))
        return PA_ERR_WORKSPACE;
    if (num_seqs == 0)
        return PA_OK;
    if (!tmp_out || !max_logits || !exp_sums)
        return PA_ERR_INVALID_ARG;
    DecodeLaunch L;
    st = prepare_decode(L, out, query, k_pool, v_pool, block_tables, max_blocks_per_seq,
                        context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                        bs_log2, num_blocks, scale, dtype, group, dev_status, stream);
    if (st != PA_OK)
        return st;
    DecodeParams &p = L.p;
    p.tmp_out = tmp_out;
    p.max_logits = max_logits;
    p.exp_sums = exp_sums;
    p.partition_size = partition_size;
    p.max_parts = max_partitions;
    p.ctx_cap = (int)std::min<int64_t>((int64_t)max_blocks_per_seq * block_size,
                                       (int64_t)max_partitions * partition_size);
    p.mode = 1;
    p.public_partials = 1;
    int grid = 0;
    st = decode_call(L, dtype, &grid, false);
    if (st != PA_OK)
        return st;
    const int64_t tiles_up =
        (int64_t)num_seqs * p.head_groups * (round_up(std::max(max_context_len, 1), 16) / 16);
    grid = (int)std::min<int64_t>(grid, tiles_up);
    st = decode_call(L, dtype, &grid, true);
    ++g_launches;
    return st;
}

pa_status pa_splitk_reduce(void *out, const float *tmp_out, const float *max_logits,
                           const float *exp_sums, const int32_t *context_lens, int num_seqs,
                           int num_q_heads, int head_dim, int partition_size,
                           int max_partitions, pa_dtype dtype, void *stream)
{
    if (num_seqs < 0 || num_q_heads <= 0 || partition_size <= 0 ||
        partition_size % pa::kTile != 0 || max_partitions <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16)
        return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0)
        return PA_OK;
    if (!out || !tmp_out || !max_logits || !exp_sums || !context_lens)
        return PA_ERR_INVALID_ARG;
    const int64_t cap = (int64_t)max_partitions * partition_size;
    return launch_reduce(out, tmp_out, max_logits, exp_sums, context_lens, num_seqs, num_q_heads,
                         head_dim, partition_size, max_partitions,
                         (int)std::min<int64_t>(cap, INT32_MAX), dtype,
                         static_cast<cudaStream_t>(stream));
}

// pa_decode_attention and pa_decode_attention_fp8 (kv8: E4M3 pools with
// scales, bf16 query and output).
static pa_status decode_entry(void *out, const void *query, const void *k_pool,
                              const void *v_pool, const int32_t *block_tables,
                              int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                              int max_context_len, int num_q_heads, int num_kv_heads,
                              int head_dim, int block_size, int64_t num_blocks, float scale,
                              pa_dtype dtype, void *workspace, size_t workspace_bytes,
                              int32_t *dev_status, void *stream, bool kv8, float k_scale,
                              float v_scale)
{
    int group = 0, bs_log2 = 0;
    pa_status st = check_attention_args(out, query, k_pool, v_pool, block_tables,
                                        max_blocks_per_seq, context_lens, num_seqs,
                                        max_context_len, num_q_heads, num_kv_heads, head_dim,
                                        block_size, num_blocks, dtype, &group, &bs_log2);
    if (st != PA_OK)
        return st;
    if (num_seqs == 0)
        return PA_OK;
    DecodeLaunch L;
    st = prepare_decode(L, out, query, k_pool, v_pool, block_tables, max_blocks_per_seq,
                        context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                        bs_log2, num_blocks, scale, dtype, group, dev_status, stream, kv8,
                        k_scale, v_scale);
    if (st != PA_OK)
        return st;
    DecodeParams &p = L.p;
    const int64_t cap_tokens = (int64_t)max_blocks_per_seq * block_size;
    p.partition_size = (int)round_up(cap_tokens, 16);   // one partition: the whole context
    p.max_parts = 1;
    p.ctx_cap = (int)cap_tokens;

    int grid = 0;
    st = decode_call(L, dtype, &grid, false);
    if (st != PA_OK)
        return st;
    const int64_t tiles_up =
        (int64_t)num_seqs * p.head_groups * (round_up(std::max(max_context_len, 1), 16) / 16);
    grid = (int)std::min<int64_t>(grid, tiles_up);
    const size_t need = stream_k_bytes(num_seqs, num_kv_heads, group, head_dim, grid);
    // a merge keeps its pieces' stats and weights, and two copy buffers of
    // piece accumulators, in a warp's share of the stage ring
    const int64_t ring_share =
        (int64_t)p.geo.spw * p.geo.stage_bytes / (p.geo.hpc * (kv8 ? pa::kSubs8 : 1)) & ~(int64_t)127;
    const bool stream_k = workspace != nullptr && workspace_bytes >= need &&
                          aligned16(workspace) &&
                          pa::merge_scratch_bytes(group, head_dim, grid) <= ring_share;
    if (stream_k) {
        p.mode = 0;
        p.slot_floats = (int)slot_floats(group, head_dim);
        p.wpart = static_cast<float *>(workspace);
        p.counters = reinterpret_cast<unsigned long long *>(
            static_cast<uint8_t *>(workspace) +
            partials_bytes((int64_t)grid * p.geo.hpc, group, head_dim));
        p.epoch = next_epoch();
    } else {
        p.mode = 1;
    }
    const int want = grid;
    st = decode_call(L, dtype, &grid, true);
    ++g_launches;
    if (st == PA_OK && stream_k && grid != want)
        return PA_ERR_CUDA;   // capacity changed between query and launch
    return st;
}

pa_status pa_decode_attention(void *out, const void *query, const void *k_pool,
                              const void *v_pool, const int32_t *block_tables,
                              int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                              int max_context_len, int num_q_heads, int num_kv_heads,
                              int head_dim, int block_size, int64_t num_blocks, float scale,
                              pa_dtype dtype, void *workspace, size_t workspace_bytes,
                              int32_t *dev_status, void *stream)
{
    return decode_entry(out, query, k_pool, v_pool, block_tables, max_blocks_per_seq,
                        context_lens, num_seqs, max_context_len, num_q_heads, num_kv_heads,
                        head_dim, block_size, num_blocks, scale, dtype, workspace,
                        workspace_bytes, dev_status, stream, false, 1.f, 1.f);
}

pa_status pa_decode_attention_fp8(void *out, const void *query, const void *k_pool,
                                  const void *v_pool, const int32_t *block_tables,
                                  int max_blocks_per_seq, const int32_t *context_lens,
                                  int num_seqs, int max_context_len, int num_q_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int64_t num_blocks, float scale, float k_scale, float v_scale,
                                  void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                  void *stream)
{
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
        return PA_ERR_INVALID_ARG;
    if ((head_dim != 128 && head_dim != 256) || (block_size != 16 && block_size != 32))
        return PA_ERR_UNSUPPORTED;
    return decode_entry(out, query, k_pool, v_pool, block_tables, max_blocks_per_seq,
                        context_lens, num_seqs, max_context_len, num_q_heads, num_kv_heads,
                        head_dim, block_size, num_blocks, scale, PA_DTYPE_BF16, workspace,
                        workspace_bytes, dev_status, stream, true, k_scale, v_scale);
}

pa_status pa_decode_attention_static(void *out, const void *query, const void *k_pool,
                                     const void *v_pool, const int32_t *block_tables,
                                     int max_blocks_per_seq, const int32_t *context_lens,
                                     int num_seqs, int max_context_len, int num_q_heads,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int64_t num_blocks, float scale, pa_dtype dtype,
                                     int32_t *dev_status, void *stream)
{
    size_t need = 0;
    pa_status st = stream_k_need(&need, out, query, k_pool, v_pool, block_tables,
                                 max_blocks_per_seq, context_lens, num_seqs, max_context_len,
                                 num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                 scale, dtype);
    if (st != PA_OK)
        return st;
    if (num_seqs == 0)
        return PA_OK;
    if (need > (size_t)PA_STATIC_SCRATCH_BYTES)
        return PA_ERR_WORKSPACE;   // these sizes need more than the fixed scratch
    void *scratch = static_scratch_address();
    if (scratch == nullptr)
        return PA_ERR_CUDA;
    return pa_decode_attention(out, query, k_pool, v_pool, block_tables, max_blocks_per_seq,
                               context_lens, num_seqs, max_context_len, num_q_heads, num_kv_heads,
                               head_dim, block_size, num_blocks, scale, dtype, scratch,
                               (size_t)PA_STATIC_SCRATCH_BYTES, dev_status, stream);
}

}  // extern "C"
