// decode.cu -- multi-sequence decode over a unified q8_0 / q4_0 KV cache.
//
// The quantised K/V blocks are never converted as a whole: each warp copies the
// raw bytes of a 32-key tile into shared memory (cp.async) and dequantises them
// into tensor-core fragments in registers right before each mma.sync
// ("unsloth llama.cpp: dequantize q4_0/q8_0 K/V tiles in the FA MMA kernel",
// summary: tiles are dequantised as they are loaded instead of a whole-cache
// f16 conversion per layer per step).
//
// Work split.  For one sequence and one kv head the g query heads x n_q new
// tokens fold into M = g*n_q <= 16 rows (fold row r = rep*n_q + t, query head
// kv*g + rep), one m16n8k16 tile high.  The sequence's cells are cut into
// `splits` chunks; one CTA of 4 warps takes one (sequence, kv head, chunk), each
// warp walking 32-key tiles of the chunk with its own online softmax.  The CTA
// merges its warps and writes one partial (max, sum, unnormalised O) per row;
// a second kernel merges the chunks by their log-sum-exp weights (the output
// merge of "TransformerEngine: FA4 in context-parallel attention", flowchart).
//
// Scores are kept in log2 units: Q is pre-multiplied by scale*log2(e) before it
// is rounded to f16.  Integer -> f16 conversion places the byte or nibble in
// the mantissa of 1024.0 (0x6400) and subtracts the offset, which is exact for
// every value a q8_0 byte or q4_0 nibble can hold.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace arc {
namespace {

constexpr int WARPS = 4;
constexpr int SUB = 32;  // keys per warp step
constexpr float LN2 = 0.6931471805599453f;

template <int KVT>
struct Fmt;
template <>
struct Fmt<ARC_KV_Q8_0> {
    static constexpr int BB = 34;
};
template <>
struct Fmt<ARC_KV_Q4_0> {
    static constexpr int BB = 18;
};

ARC_DEV void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

ARC_DEV uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
ARC_DEV __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// Bytes 0 and 1 of x (signed int8) -> half2 of the same integers.
ARC_DEV __half2 s8x2_to_h2(uint32_t x)
{
    const uint32_t v = __byte_perm(x ^ 0x8080u, 0x64646464u, 0x4140u);
    return __hsub2(bits_h2(v), bits_h2(0x64806480u));  // 1024 + 128
}

// Bytes 0 and 1 of x, each holding a value 0..15 -> half2 of (n - 8).
ARC_DEV __half2 u4x2_to_h2(uint32_t x)
{
    const uint32_t v = __byte_perm(x, 0x64646464u, 0x4140u);
    return __hsub2(bits_h2(v), bits_h2(0x64086408u));  // 1024 + 8
}

ARC_DEV uint32_t lds_u16(const uint8_t *p) { return *reinterpret_cast<const uint16_t *>(p); }
ARC_DEV __half lds_h(const uint8_t *p) { return *reinterpret_cast<const __half *>(p); }

// K fragment (B operand of S = Q K^T): key row `row`, dims ks*16 + {2tq,2tq+1} and +8.
template <int KVT>
ARC_DEV void k_frag(const uint8_t *row, int ks, int tq, uint32_t &b0, uint32_t &b1)
{
    const int blk = ks >> 1;
    const uint8_t *bp = row + blk * Fmt<KVT>::BB;
    const __half2 sc = __half2half2(lds_h(bp));
    if constexpr (KVT == ARC_KV_Q8_0) {
        const int e0 = (ks & 1) * 16 + 2 * tq;
        b0 = h2_bits(__hmul2(s8x2_to_h2(lds_u16(bp + 2 + e0)), sc));
        b1 = h2_bits(__hmul2(s8x2_to_h2(lds_u16(bp + 2 + e0 + 8)), sc));
    } else {
        const uint32_t x0 = lds_u16(bp + 2 + 2 * tq), x1 = lds_u16(bp + 2 + 2 * tq + 8);
        const int sh = (ks & 1) * 4;  // elements 16..31 sit in the high nibbles
        b0 = h2_bits(__hmul2(u4x2_to_h2((x0 >> sh) & 0x0F0Fu), sc));
        b1 = h2_bits(__hmul2(u4x2_to_h2((x1 >> sh) & 0x0F0Fu), sc));
    }
}

// One dequantised element d of a row, as raw integer byte (in bits 0..7) and scale.
template <int KVT>
ARC_DEV uint32_t v_code(const uint8_t *row, int d)
{
    const uint8_t *bp = row + (d >> 5) * Fmt<KVT>::BB;
    const int e = d & 31;
    if constexpr (KVT == ARC_KV_Q8_0) {
        return bp[2 + e];
    } else {
        const uint32_t byte = bp[2 + (e & 15)];
        return (e < 16) ? (byte & 15u) : (byte >> 4);
    }
}

template <int KVT>
ARC_DEV __half v_scale(const uint8_t *row, int d)
{
    return lds_h(row + (d >> 5) * Fmt<KVT>::BB);
}

// V fragment (B operand of O += P V): keys k0, k0+1 (b0) and k0+8, k0+9 (b1), dim d.
template <int KVT>
ARC_DEV void v_frag(const uint8_t *sv, int rowb, int k0, int d, uint32_t &b0, uint32_t &b1)
{
    const uint8_t *r0 = sv + (k0)*rowb, *r1 = sv + (k0 + 1) * rowb;
    const uint8_t *r8 = sv + (k0 + 8) * rowb, *r9 = sv + (k0 + 9) * rowb;
    const uint32_t x01 = v_code<KVT>(r0, d) | (v_code<KVT>(r1, d) << 8);
    const uint32_t x89 = v_code<KVT>(r8, d) | (v_code<KVT>(r9, d) << 8);
    const __half2 s01 = __halves2half2(v_scale<KVT>(r0, d), v_scale<KVT>(r1, d));
    const __half2 s89 = __halves2half2(v_scale<KVT>(r8, d), v_scale<KVT>(r9, d));
    if constexpr (KVT == ARC_KV_Q8_0) {
        b0 = h2_bits(__hmul2(s8x2_to_h2(x01), s01));
        b1 = h2_bits(__hmul2(s8x2_to_h2(x89), s89));
    } else {
        b0 = h2_bits(__hmul2(u4x2_to_h2(x01), s01));
        b1 = h2_bits(__hmul2(u4x2_to_h2(x89), s89));
    }
}

template <int BYTES>
ARC_DEV void cp_async(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(smem_u32(dst)), "l"(src), "n"(BYTES) : "memory");
}
ARC_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
ARC_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int KVT, int D>
__global__ void __launch_bounds__(WARPS * 32) decode_split_kernel(const __grid_constant__ DecodeParams p)
{
    constexpr int ROWB = (D / 32) * Fmt<KVT>::BB;   // bytes of one head row
    constexpr int TILE = SUB * ROWB;                 // bytes of one 32-key raw tile
    constexpr int KS = D / 16;                       // k-steps of S
    constexpr int NT_O = D / 8;                      // n-tiles of O
    constexpr int PIECE = (ROWB % 8 == 0) ? 8 : 4;   // cp.async granule (rows are 4-byte multiples)
    static_assert(ROWB % 4 == 0, "rows are copied in 4- or 8-byte pieces");

    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;

    const int per_seq = p.Hkv * p.splits;
    const int s = blockIdx.x / per_seq;
    const int kvh = (blockIdx.x / p.splits) % p.Hkv;
    const int sp = blockIdx.x % p.splits;
    const arc_seq sq = p.seqs[s];
    const int G = p.H / p.Hkv;
    const int M = G * sq.n_q;
    const int c_begin = sp * p.chunk;
    const int c_end = min(c_begin + p.chunk, sq.n_kv);
    const int64_t part = (int64_t)blockIdx.x;

    // ---- Q fragments (16 rows x D), pre-scaled into log2 units, f16
    uint32_t qa[KS][4];
    int row_t[2];  // token index within the sequence for rows g and g+8 (-1: padding row)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int r = g + 8 * hr;
        row_t[hr] = (r < M) ? r % sq.n_q : -1;
    }
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int part_i = 0; part_i < 4; ++part_i) {
            const int r = g + 8 * (part_i & 1);
            const int d = ks * 16 + 2 * tq + 8 * (part_i >> 1);
            float2 v = make_float2(0.f, 0.f);
            if (r < M) {
                const int h = kvh * G + r / sq.n_q;
                const int tok = sq.q_begin + r % sq.n_q;
                v = *reinterpret_cast<const float2 *>(p.q + ((int64_t)tok * p.H + h) * D + d);
            }
            qa[ks][part_i] = h2_bits(__floats2half2_rn(v.x * p.scale_log2, v.y * p.scale_log2));
        }
    }

    float o[NT_O][4];
#pragma unroll
    for (int i = 0; i < NT_O; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};

    uint8_t *wbuf = smem + warp * (4 * TILE);  // [stage 2][K,V] tiles of this warp
    const int n_steps = c_end > c_begin ? (c_end - c_begin + SUB - 1) / SUB : 0;
    const int my_steps = n_steps > warp ? (n_steps - warp + WARPS - 1) / WARPS : 0;
    const uint8_t *kbase = p.k_cache + (int64_t)kvh * ROWB;
    const uint8_t *vbase = p.v_cache + (int64_t)kvh * ROWB;
    const int64_t cell_stride = (int64_t)p.Hkv * ROWB;

    auto issue = [&](int i, int stage) {
        const int key0 = c_begin + (warp + i * WARPS) * SUB;
        uint8_t *dk = wbuf + stage * 2 * TILE;
        uint8_t *dv = dk + TILE;
        for (int x = lane; x < SUB * (ROWB / PIECE); x += 32) {
            const int kr = x / (ROWB / PIECE), off = (x % (ROWB / PIECE)) * PIECE;
            const int key = min(key0 + kr, c_end - 1);  // rows past the chunk repeat a valid row; masked
            const int64_t cell = sq.kv_begin + key;
            cp_async<PIECE>(dk + kr * ROWB + off, kbase + cell * cell_stride + off);
            cp_async<PIECE>(dv + kr * ROWB + off, vbase + cell * cell_stride + off);
        }
        cp_async_commit();
    };

    if (my_steps > 0) issue(0, 0);
    for (int i = 0; i < my_steps; ++i) {
        const int stage = i & 1;
        if (i + 1 < my_steps) {
            issue(i + 1, stage ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        const uint8_t *sk = wbuf + stage * 2 * TILE;
        const uint8_t *sv = sk + TILE;
        const int key0 = c_begin + (warp + i * WARPS) * SUB;

        // ---- S = Q K^T for 32 keys: 4 n-tiles of 8 keys
        float sacc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
            const uint8_t *krow = sk + (nt * 8 + g) * ROWB;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t b0, b1;
                k_frag<KVT>(krow, ks, tq, b0, b1);
                mma16816(sacc[nt], qa[ks], b0, b1);
            }
        }
        // ---- mask: key index vs. the chunk end and each row's causal limit
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int lim = row_t[hr] < 0 ? -1 : sq.n_kv - sq.n_q + row_t[hr];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int key = key0 + nt * 8 + 2 * tq + e;
                    if (key >= c_end || key > lim) sacc[nt][2 * hr + e] = -INFINITY;
                }
        }
        // ---- online softmax for rows g and g+8 (a row is spread over the 4 lanes of a quad)
        uint32_t pa[2][4];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) mx = fmaxf(mx, fmaxf(sacc[nt][2 * hr], sacc[nt][2 * hr + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_r[hr], mx);
            const float msafe = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = (m_r[hr] == -INFINITY) ? 0.f : fast_exp2(m_r[hr] - msafe);
            m_r[hr] = m_new;
            float rs = 0.f;
            float pv[4][2];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    pv[nt][e] = fast_exp2(sacc[nt][2 * hr + e] - msafe);
                    rs += pv[nt][e];
                }
            l_r[hr] = l_r[hr] * alpha + rs;
#pragma unroll
            for (int i2 = 0; i2 < NT_O; ++i2) {
                o[i2][2 * hr] *= alpha;
                o[i2][2 * hr + 1] *= alpha;
            }
            // A fragments of P for the two 16-key k-steps
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                pa[kk][hr] = h2_bits(__floats2half2_rn(pv[2 * kk][0], pv[2 * kk][1]));
                pa[kk][2 + hr] = h2_bits(__floats2half2_rn(pv[2 * kk + 1][0], pv[2 * kk + 1][1]));
            }
        }
        // ---- O += P V
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
            for (int nd = 0; nd < NT_O; ++nd) {
                uint32_t b0, b1;
                v_frag<KVT>(sv, ROWB, kk * 16 + 2 * tq, nd * 8 + g, b0, b1);
                mma16816(o[nd], pa[kk], b0, b1);
            }
        }
        __syncwarp();
    }

    // ---- merge the 4 warps of this CTA in shared memory
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 1);
        l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 2);
    }
    __syncthreads();  // all warps are done with their raw tiles
    float *so = reinterpret_cast<float *>(smem);       // [WARPS][16][D]
    float *sml = so + WARPS * 16 * D;                   // [WARPS][16][2]
#pragma unroll
    for (int nd = 0; nd < NT_O; ++nd)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            float *dst = so + ((warp * 16) + g + 8 * hr) * D + nd * 8 + 2 * tq;
            dst[0] = o[nd][2 * hr];
            dst[1] = o[nd][2 * hr + 1];
        }
    if (tq == 0) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            sml[(warp * 16 + g + 8 * hr) * 2 + 0] = m_r[hr];
            sml[(warp * 16 + g + 8 * hr) * 2 + 1] = l_r[hr];
        }
    }
    __syncthreads();
    for (int x = threadIdx.x; x < 16 * D; x += WARPS * 32) {
        const int r = x / D, d = x % D;
        float mm = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) mm = fmaxf(mm, sml[(w * 16 + r) * 2]);
        const float ms = (mm == -INFINITY) ? 0.f : mm;
        float acc = 0.f, ll = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float mw = sml[(w * 16 + r) * 2];
            const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - ms);
            acc += f * so[(w * 16 + r) * D + d];
            ll += f * sml[(w * 16 + r) * 2 + 1];
        }
        p.ws_o[(part * 16 + r) * D + d] = acc;
        if (d == 0) {
            p.ws_ml[(part * 16 + r) * 2 + 0] = mm;
            p.ws_ml[(part * 16 + r) * 2 + 1] = ll;
        }
    }
}

// Merge the chunk partials of one (sequence, kv head, fold row) by their
// log-sum-exp weights, normalise, write O and LSE.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const __grid_constant__ DecodeParams p)
{
    const int s = blockIdx.x / p.Hkv, kvh = blockIdx.x % p.Hkv, r = blockIdx.y;
    const arc_seq sq = p.seqs[s];
    const int G = p.H / p.Hkv;
    if (r >= G * sq.n_q) return;
    const int h = kvh * G + r / sq.n_q, tok = sq.q_begin + r % sq.n_q;
    const int d = threadIdx.x;
    const int64_t part0 = ((int64_t)s * p.Hkv + kvh) * p.splits;
    float mm = -INFINITY;
    for (int sp = 0; sp < p.splits; ++sp) mm = fmaxf(mm, p.ws_ml[((part0 + sp) * 16 + r) * 2]);
    const float ms = (mm == -INFINITY) ? 0.f : mm;
    float acc = 0.f, ll = 0.f;
    for (int sp = 0; sp < p.splits; ++sp) {
        const float mw = p.ws_ml[((part0 + sp) * 16 + r) * 2];
        if (mw == -INFINITY) continue;
        const float f = exp2f(mw - ms);
        acc += f * p.ws_o[((part0 + sp) * 16 + r) * D + d];
        ll += f * p.ws_ml[((part0 + sp) * 16 + r) * 2 + 1];
    }
    p.o[((int64_t)tok * p.H + h) * D + d] = ll > 0.f ? acc / ll : 0.f;
    if (d == 0) p.lse[(int64_t)tok * p.H + h] = ll > 0.f ? (mm + log2f(ll)) * LN2 : -INFINITY;
}

template <int KVT, int D>
cudaError_t launch_t(const DecodeParams &p, cudaStream_t s)
{
    constexpr int ROWB = (D / 32) * Fmt<KVT>::BB;
    const int tiles = WARPS * 4 * SUB * ROWB;
    const int merge = WARPS * 16 * (D + 2) * 4;
    const int smem = tiles > merge ? tiles : merge;
    auto k1 = decode_split_kernel<KVT, D>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = p.n_seq * p.Hkv * p.splits;
    if (grid == 0) return cudaSuccess;
    k1<<<grid, WARPS * 32, smem, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    decode_combine_kernel<D><<<dim3(p.n_seq * p.Hkv, 16), D, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

int decode_smem_bytes(int kv_type, int D)
{
    const int bb = kv_type == ARC_KV_Q8_0 ? 34 : 18;
    const int tiles = WARPS * 4 * SUB * (D / 32) * bb;
    const int merge = WARPS * 16 * (D + 2) * 4;
    return tiles > merge ? tiles : merge;
}

cudaError_t launch_decode(const DecodeParams &p, cudaStream_t s)
{
    if (p.kv_type == ARC_KV_Q8_0) {
        if (p.D == 64) return launch_t<ARC_KV_Q8_0, 64>(p, s);
        if (p.D == 128) return launch_t<ARC_KV_Q8_0, 128>(p, s);
    } else {
        if (p.D == 64) return launch_t<ARC_KV_Q4_0, 64>(p, s);
        if (p.D == 128) return launch_t<ARC_KV_Q4_0, 128>(p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace arc
