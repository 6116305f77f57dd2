// merge.cu -- merge of partial attention results over disjoint key sets.
//
// "TransformerEngine: FA4 in context-parallel attention" (flowchart): with the
// keys of a row split over parts, part i gives a normalised O_i and LSE_i, and
//     LSE = ln( sum_i exp(LSE_i) [+ exp(sink)] ),   O = sum_i exp(LSE_i - LSE) O_i
// is attention over all the keys.  One warp per row: the lanes read the parts'
// LSE values (a broadcast), every lane forms the weights itself, and each lane
// then owns pairs of columns (2 * lane, 2 * lane + 64, ...), reading every part
// before writing, so o may alias o_parts[0].  HBM-bound: each part's row is read
// once and the output row written once.
#include <math.h>

#include "internal.h"

namespace arc {
namespace {

template <typename T>
struct Pair;
template <>
struct Pair<float> {
    static __device__ __forceinline__ float2 load(const void *p, int64_t i)
    {
        return *reinterpret_cast<const float2 *>(static_cast<const float *>(p) + i);
    }
    static __device__ __forceinline__ void store(void *p, int64_t i, float2 v)
    {
        *reinterpret_cast<float2 *>(static_cast<float *>(p) + i) = v;
    }
};
template <>
struct Pair<__nv_bfloat16> {
    static __device__ __forceinline__ float2 load(const void *p, int64_t i)
    {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(static_cast<const __nv_bfloat16 *>(p) + i));
    }
    static __device__ __forceinline__ void store(void *p, int64_t i, float2 v)
    {
        *reinterpret_cast<__nv_bfloat162 *>(static_cast<__nv_bfloat16 *>(p) + i) = __float22bfloat162_rn(v);
    }
};

constexpr int MERGE_ROWS_PER_CTA = 8;   // one warp per row

template <typename T>
__global__ void __launch_bounds__(32 * MERGE_ROWS_PER_CTA) merge_kernel(const __grid_constant__ MergeParams p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * MERGE_ROWS_PER_CTA + warp;
    if (r >= p.rows) return;
    const int n = p.n_parts;

    float l[ARC_MERGE_MAX_PARTS];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < ARC_MERGE_MAX_PARTS; ++i) {
        l[i] = i < n ? p.lse_parts[i][r] : -INFINITY;
        mx = fmaxf(mx, l[i]);
    }
    const float sink = p.sinks ? p.sinks[(r / p.sink_rows) % p.sink_heads] : -INFINITY;
    mx = fmaxf(mx, sink);
    float lse = -INFINITY;
    float w[ARC_MERGE_MAX_PARTS];
    if (mx == -INFINITY) {
#pragma unroll
        for (int i = 0; i < ARC_MERGE_MAX_PARTS; ++i) w[i] = 0.f;
    } else {
        float sum = (sink == -INFINITY) ? 0.f : expf(sink - mx);
#pragma unroll
        for (int i = 0; i < ARC_MERGE_MAX_PARTS; ++i) sum += (l[i] == -INFINITY) ? 0.f : expf(l[i] - mx);
        lse = mx + logf(sum);
#pragma unroll
        for (int i = 0; i < ARC_MERGE_MAX_PARTS; ++i) w[i] = (l[i] == -INFINITY) ? 0.f : expf(l[i] - lse);
    }
    __syncwarp();   // every lane has read lse_parts[.][r] before lane 0 may overwrite an aliased lse
    if (lane == 0) p.lse[r] = lse;

    const int64_t base = (int64_t)r * p.dv;
    for (int d = 2 * lane; d < p.dv; d += 64) {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < ARC_MERGE_MAX_PARTS; ++i) {
            if (i < n && w[i] != 0.f) {
                const float2 v = Pair<T>::load(p.o_parts[i], base + d);
                acc.x += w[i] * v.x, acc.y += w[i] * v.y;
            }
        }
        Pair<T>::store(p.o, base + d, acc);
    }
}

}  // namespace

cudaError_t launch_merge(const MergeParams &p, cudaStream_t s)
{
    if (p.rows == 0) return cudaSuccess;
    const int grid = (p.rows + MERGE_ROWS_PER_CTA - 1) / MERGE_ROWS_PER_CTA;
    if (p.dtype == ARC_DTYPE_F32)
        merge_kernel<float><<<grid, 32 * MERGE_ROWS_PER_CTA, 0, s>>>(p);
    else
        merge_kernel<__nv_bfloat16><<<grid, 32 * MERGE_ROWS_PER_CTA, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace arc
