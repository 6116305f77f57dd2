// merge.cu -- merge of partial attention results over disjoint key sets.
//
// "TransformerEngine: FA4 in context-parallel attention" (flowchart): with the
// keys of a row split over parts, part i gives a normalised O_i and LSE_i, and
//     LSE = ln( sum_i exp(LSE_i) [+ exp(sink)] ),   O = sum_i exp(LSE_i - LSE) O_i
// is attention over all the keys.  One warp per row: the lanes read the parts'
// LSE values (a broadcast) and every lane forms the weights itself.  Each lane
// then owns 8-element chunks of the row (chunk lane, lane + 32, ...; 16-byte
// loads, up to four chunks in flight per part), reading every part before it
// writes, so o may alias o_parts[0].  Rows whose pointers or width do not allow
// 16-byte accesses take a 2-element path.  HBM-bound: each part's row is read
// once and the output row written once.
#include <math.h>

#include <type_traits>

#include "internal.h"

namespace arc {
namespace {

// Eight consecutive elements as fp32, and back.
template <typename T>
struct Oct;
template <>
struct Oct<float> {
    static __device__ __forceinline__ void load(const void *p, int64_t i, float (&v)[8])
    {
        const float4 *q = reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
        const float4 a = q[0], b = q[1];
        v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
    }
    static __device__ __forceinline__ void store(void *p, int64_t i, const float (&v)[8])
    {
        float4 *q = reinterpret_cast<float4 *>(static_cast<float *>(p) + i);
        q[0] = make_float4(v[0], v[1], v[2], v[3]);
        q[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
};
template <>
struct Oct<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const void *p, int64_t i, float (&v)[8])
    {
        const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p) + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
            v[2 * k] = f.x, v[2 * k + 1] = f.y;
        }
    }
    static __device__ __forceinline__ void store(void *p, int64_t i, const float (&v)[8])
    {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const __nv_bfloat162 h = __float22bfloat162_rn(make_float2(v[2 * k], v[2 * k + 1]));
            w[k] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p) + i) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

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

// NP: a compile-time bound on the number of parts (the loops over parts unroll to it).
// T: the parts' element type; TO: the output's (the same, or bf16 from fp32 partials).
template <typename T, typename TO, bool VEC, int NP>
__global__ void __launch_bounds__(32 * MERGE_ROWS_PER_CTA) merge_kernel(const __grid_constant__ MergeParams p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * MERGE_ROWS_PER_CTA + warp;
    if (r >= p.rows) return;
    const int n = p.n_parts;

    float l[NP];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        l[i] = i < n ? p.lse_parts[i][r] : -INFINITY;
        mx = fmaxf(mx, l[i]);
    }
    const float sink = p.sinks ? p.sinks[(r / p.sink_rows) % p.sink_heads] : -INFINITY;
    mx = fmaxf(mx, sink);
    float lse = -INFINITY;
    float w[NP];
    if (mx == -INFINITY) {
#pragma unroll
        for (int i = 0; i < NP; ++i) w[i] = 0.f;
    } else {
        float sum = (sink == -INFINITY) ? 0.f : expf(sink - mx);
#pragma unroll
        for (int i = 0; i < NP; ++i) sum += (l[i] == -INFINITY) ? 0.f : expf(l[i] - mx);
        lse = mx + logf(sum);
#pragma unroll
        for (int i = 0; i < NP; ++i) w[i] = (l[i] == -INFINITY) ? 0.f : expf(l[i] - lse);
    }
    __syncwarp();   // every lane has read lse_parts[.][r] before lane 0 may overwrite an aliased lse
    if (lane == 0) p.lse[r] = lse;

    const int64_t base = (int64_t)r * p.dv;
    if constexpr (VEC) {
        constexpr int U = 2;                        // chunks of a lane per pass (d_v 512: one pass)
        const int nch = p.dv / 8;
        for (int c0 = lane; c0 < nch; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                if (i < n && w[i] != 0.f) {
                    float v[U][8];
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (c0 + 32 * u < nch) Oct<T>::load(p.o_parts[i], base + 8 * (c0 + 32 * u), v[u]);
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (c0 + 32 * u < nch)
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[u][e] += w[i] * v[u][e];
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c0 + 32 * u < nch) Oct<TO>::store(p.o, base + 8 * (c0 + 32 * u), acc[u]);
        }
    } else {
        for (int d = 2 * lane; d < p.dv; d += 64) {
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                if (i < n && w[i] != 0.f) {
                    const float2 v = Pair<T>::load(p.o_parts[i], base + d);
                    acc.x += w[i] * v.x, acc.y += w[i] * v.y;
                }
            }
            Pair<TO>::store(p.o, base + d, acc);
        }
    }
}

}  // namespace

cudaError_t launch_merge(const MergeParams &p, cudaStream_t s)
{
    if (p.rows == 0) return cudaSuccess;
    const int grid = (p.rows + MERGE_ROWS_PER_CTA - 1) / MERGE_ROWS_PER_CTA;
    // 16-byte path: every row starts 16-byte aligned (dv a multiple of 8 elements, bases aligned)
    bool vec = p.dv % 8 == 0 && (reinterpret_cast<uintptr_t>(p.o) & 15) == 0;
    for (int i = 0; i < p.n_parts; ++i) vec = vec && (reinterpret_cast<uintptr_t>(p.o_parts[i]) & 15) == 0;
    const dim3 block(32 * MERGE_ROWS_PER_CTA);
    auto go = [&](auto np) {
        constexpr int NP = decltype(np)::value;
        if (p.dtype == ARC_DTYPE_F32 && p.out_dtype == ARC_DTYPE_F32) {
            if (vec)
                merge_kernel<float, float, true, NP><<<grid, block, 0, s>>>(p);
            else
                merge_kernel<float, float, false, NP><<<grid, block, 0, s>>>(p);
        } else if (p.dtype == ARC_DTYPE_F32) {
            if (vec)
                merge_kernel<float, __nv_bfloat16, true, NP><<<grid, block, 0, s>>>(p);
            else
                merge_kernel<float, __nv_bfloat16, false, NP><<<grid, block, 0, s>>>(p);
        } else {
            if (vec)
                merge_kernel<__nv_bfloat16, __nv_bfloat16, true, NP><<<grid, block, 0, s>>>(p);
            else
                merge_kernel<__nv_bfloat16, __nv_bfloat16, false, NP><<<grid, block, 0, s>>>(p);
        }
    };
    if (p.n_parts <= 2)
        go(std::integral_constant<int, 2>{});
    else if (p.n_parts <= 4)
        go(std::integral_constant<int, 4>{});
    else
        go(std::integral_constant<int, ARC_MERGE_MAX_PARTS>{});
    return cudaGetLastError();
}

}  // namespace arc
