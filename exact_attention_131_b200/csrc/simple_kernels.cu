// simple_kernels.cu -- CUDA-core attention kernels: one warp per output row, the
// 32 lanes splitting the head dims, keys visited one at a time with an online
// softmax in fp32.  They serve the fp32 reference mode (no tensor cores, no
// TF32) and the control arm that the engagement tests compare the tensor-core
// kernels against.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace arc {
namespace {

constexpr int kMaxChunks = 16;  // head dims up to 512 = 16 x 32 lanes

template <typename T>
__device__ __forceinline__ float ld(const void *base, int64_t off);
template <>
__device__ __forceinline__ float ld<float>(const void *base, int64_t off)
{
    return static_cast<const float *>(base)[off];
}
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const void *base, int64_t off)
{
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(base)[off]);
}
template <typename T>
__device__ __forceinline__ void st(void *base, int64_t off, float v);
template <>
__device__ __forceinline__ void st<float>(void *base, int64_t off, float v)
{
    static_cast<float *>(base)[off] = v;
}
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(void *base, int64_t off, float v)
{
    static_cast<__nv_bfloat16 *>(base)[off] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Online-softmax state of one row, replicated in all 32 lanes.
struct RowState {
    float m = -INFINITY, l = 0.f;
    float acc[kMaxChunks];
};

__device__ __forceinline__ void row_update(RowState &st_, float s, const float (&v)[kMaxChunks], int nv)
{
    float m_new = fmaxf(st_.m, s);
    float alpha = (st_.m == -INFINITY) ? 0.f : expf(st_.m - m_new);
    float p = expf(s - m_new);
    st_.l = st_.l * alpha + p;
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i)
        if (i < nv) st_.acc[i] = st_.acc[i] * alpha + p * v[i];
    st_.m = m_new;
}

template <typename T>
__global__ void simple_attn_kernel(SimpleParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int nq = (p.Dqk + 31) / 32, nv = (p.Dv + 31) / 32;
    // rows: dense/MLA (b, h, t); sparse (t, h)
    int64_t total = (p.mode == 2) ? (int64_t)p.Tq * p.H : (int64_t)p.B * p.H * p.Tq;
    if (row >= total) return;
    int b = 0, h, t;
    if (p.mode == 2) {
        t = (int)(row / p.H);
        h = (int)(row % p.H);
    } else {
        b = (int)(row / ((int64_t)p.H * p.Tq));
        h = (int)((row / p.Tq) % p.H);
        t = (int)(row % p.Tq);
    }
    const int kvh = (p.mode == 0) ? h / (p.H / p.Hkv) : h;

    float q[kMaxChunks];
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) {
        q[i] = 0.f;
        int d = lane + 32 * i;
        if (i < nq && d < p.Dqk) {
            if (p.mode == 0)
                q[i] = ld<T>(p.q, b * p.qs[0] + h * p.qs[1] + t * p.qs[2] + d);
            else if (p.mode == 1)
                q[i] = d < p.Dn ? ld<T>(p.q, b * p.qs[0] + h * p.qs[1] + t * p.qs[2] + d)
                                : ld<T>(p.q2, b * p.q2s[0] + h * p.q2s[1] + t * p.q2s[2] + (d - p.Dn));
            else
                q[i] = ld<T>(p.q, t * p.qs[0] + h * p.qs[1] + d);
        }
    }

    RowState rs;
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) rs.acc[i] = 0.f;

    const int n_keys = (p.mode == 2) ? p.topk : p.Tk;
    int last = n_keys - 1;
    if (p.mode != 2 && p.causal) last = min(last, t + (p.Tk - p.Tq));
    for (int j = 0; j <= last; ++j) {
        int64_t key = j;
        if (p.mode == 2) {
            key = p.idx[(int64_t)t * p.idx_stride + j];
            if (key < 0 || key >= p.Skv) continue;
        }
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxChunks; ++i) {
            int d = lane + 32 * i;
            if (i < nq && d < p.Dqk) {
                float kval;
                if (p.mode == 0)
                    kval = ld<T>(p.k, b * p.ks[0] + kvh * p.ks[1] + key * p.ks[2] + d);
                else if (p.mode == 1)
                    kval = d < p.Dn ? ld<T>(p.k, b * p.ks[0] + kvh * p.ks[1] + key * p.ks[2] + d)
                                    : ld<T>(p.k2, b * p.k2s[0] + key * p.k2s[1] + (d - p.Dn));
                else
                    kval = ld<T>(p.k, key * p.ks[0] + d);
                part += q[i] * kval;
            }
        }
        float s = warp_sum(part) * p.scale;
        float v[kMaxChunks];
#pragma unroll
        for (int i = 0; i < kMaxChunks; ++i) {
            v[i] = 0.f;
            int d = lane + 32 * i;
            if (i < nv && d < p.Dv) {
                if (p.mode == 2)
                    v[i] = p.v ? ld<T>(p.v, key * p.vs[0] + d) : ld<T>(p.k, key * p.ks[0] + d);
                else
                    v[i] = ld<T>(p.v, b * p.vs[0] + kvh * p.vs[1] + key * p.vs[2] + d);
            }
        }
        row_update(rs, s, v, nv);
    }

    // Sink: one extra term in the denominator only.
    float m = rs.m, l = rs.l, fac;
    if (p.sinks) {
        float sg = p.sinks[h];
        float mf = fmaxf(m, sg);
        float a = (m == -INFINITY) ? 0.f : expf(m - mf);
        l = l * a + expf(sg - mf);
        fac = a / l;
        m = mf;
    } else {
        fac = (l > 0.f) ? 1.f / l : 0.f;
    }
    int64_t obase = (p.mode == 2) ? t * p.os[0] + h * p.os[1] : b * p.os[0] + h * p.os[1] + t * p.os[2];
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) {
        int d = lane + 32 * i;
        if (i < nv && d < p.Dv) st<T>(p.o, obase + d, rs.acc[i] * fac);
    }
    if (lane == 0) p.lse[row] = (l > 0.f) ? m + logf(l) : -INFINITY;
}

// ---------------------------------------------------------------- decode

__device__ __forceinline__ float dequant(int kv_type, const uint8_t *row, int d)
{
    int blk = d >> 5, e = d & 31;
    if (kv_type == ARC_KV_Q8_0) {
        const uint8_t *bp = row + blk * 34;
        float sc = __half2float(*reinterpret_cast<const __half *>(bp));
        return sc * (float)(int8_t)bp[2 + e];
    }
    const uint8_t *bp = row + blk * 18;
    float sc = __half2float(*reinterpret_cast<const __half *>(bp));
    int n = (e < 16) ? (bp[2 + e] & 15) : (bp[2 + e - 16] >> 4);
    return sc * (float)(n - 8);
}

__global__ void simple_decode_kernel(SimpleDecodeParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (row >= (int64_t)p.n_tok * p.H) return;
    const int tok = (int)(row / p.H), h = (int)(row % p.H);
    int s = -1;
    for (int i = 0; i < p.n_seq; ++i)
        if (tok >= p.seqs[i].q_begin && tok < p.seqs[i].q_begin + p.seqs[i].n_q) s = i;
    if (s < 0) return;
    const arc_seq sq = p.seqs[s];
    const int t = tok - sq.q_begin, kvh = h / (p.H / p.Hkv);
    const int nv = p.D / 32;
    const int bb = (p.kv_type == ARC_KV_Q8_0) ? 34 : 18;
    const int64_t rowb = (int64_t)(p.D / 32) * bb;
    float q[kMaxChunks];
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) q[i] = (i < nv) ? p.q[row * p.D + lane + 32 * i] : 0.f;
    RowState rs;
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) rs.acc[i] = 0.f;
    const int last = sq.n_kv - sq.n_q + t;
    for (int c = 0; c <= last; ++c) {
        const int64_t cell = sq.kv_begin + c;
        const uint8_t *kr = p.k_cache + (cell * p.Hkv + kvh) * rowb;
        const uint8_t *vr = p.v_cache + (cell * p.Hkv + kvh) * rowb;
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxChunks; ++i)
            if (i < nv) part += q[i] * dequant(p.kv_type, kr, lane + 32 * i);
        float sc = warp_sum(part) * p.scale;
        float v[kMaxChunks];
#pragma unroll
        for (int i = 0; i < kMaxChunks; ++i) v[i] = (i < nv) ? dequant(p.kv_type, vr, lane + 32 * i) : 0.f;
        row_update(rs, sc, v, nv);
    }
    float fac = rs.l > 0.f ? 1.f / rs.l : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i)
        if (i < nv) p.o[row * p.D + lane + 32 * i] = rs.acc[i] * fac;
    if (lane == 0) p.lse[row] = rs.l > 0.f ? rs.m + logf(rs.l) : -INFINITY;
}

__global__ void selftest_timeout_kernel(uint32_t *status, uint64_t timeout_ns)
{
    __shared__ alignas(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Nothing ever arrives: the bounded wait must give up and report.
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, timeout_ns)) report(status, ST_TIMEOUT_SELFTEST);
    __syncthreads();
}

}  // namespace

cudaError_t launch_simple_attn(const SimpleParams &p, cudaStream_t s)
{
    int64_t rows = (p.mode == 2) ? (int64_t)p.Tq * p.H : (int64_t)p.B * p.H * p.Tq;
    if (rows == 0) return cudaSuccess;
    const int warps = 4;
    dim3 grid((unsigned)((rows + warps - 1) / warps));
    if (p.dtype == ARC_DTYPE_F32)
        simple_attn_kernel<float><<<grid, warps * 32, 0, s>>>(p);
    else
        simple_attn_kernel<__nv_bfloat16><<<grid, warps * 32, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_simple_decode(const SimpleDecodeParams &p, cudaStream_t s)
{
    int64_t rows = (int64_t)p.n_tok * p.H;
    if (rows == 0) return cudaSuccess;
    const int warps = 4;
    simple_decode_kernel<<<(unsigned)((rows + warps - 1) / warps), warps * 32, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(uint32_t *status, uint64_t timeout_ns, cudaStream_t s)
{
    selftest_timeout_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace arc
