// decode.cu -- multi-sequence decode over a unified q8_0 / q4_0 KV cache.
//
// The quantised K/V blocks are never converted as a whole: each CTA copies the
// raw bytes of a 64-key tile into shared memory (cp.async, two stages in
// flight), and one cooperative pass turns that tile into f16 right before the
// tensor cores read it ("unsloth llama.cpp: dequantize q4_0/q8_0 K/V tiles in
// the FA MMA kernel", summary: tiles are dequantised as they are loaded
// instead of a whole-cache f16 conversion per layer per step).  Each element
// is dequantised exactly once; the f16 tile is read with ldmatrix (K) and
// ldmatrix.trans (V) into mma.sync fragments.
//
// Work split.  For one sequence and one kv head the g query heads x n_q new
// tokens fold into M = g*n_q <= 16 rows (fold row r = rep*n_q + t, query head
// kv*g + rep), one m16n8k16 tile high.  The sequence's cells are cut into
// `splits` chunks; one CTA of 4 warps takes one (sequence, kv head, chunk),
// each warp taking 16 keys of every 64-key tile with its own online softmax.
// The CTA merges its warps and writes one partial (max, sum, unnormalised O)
// per row; a second kernel, launched as a programmatic dependent of the first,
// merges the chunks by their log-sum-exp weights (the output merge of
// "TransformerEngine: FA4 in context-parallel attention", flowchart).
//
// Scores are kept in log2 units: Q is pre-multiplied by scale*log2(e) before it
// is rounded to f16.  Integer -> f16 conversion places the byte or nibble in
// the mantissa of 1024.0 (0x6400) and subtracts the offset, which is exact for
// every value a q8_0 byte or q4_0 nibble can hold; the block scale multiplies
// afterwards.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace arc {
namespace {

constexpr int WARPS = 4;
constexpr int DT = 64;             // keys per CTA tile (16 per warp)
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

constexpr int gcd16(int x) { return (x & 15) == 0 ? 16 : ((x & 7) == 0 ? 8 : ((x & 3) == 0 ? 4 : ((x & 1) == 0 ? 2 : 1))); }

// TMA: the head row of kv head h starts at byte ROWB*h of a cell, which is not
// 16-byte aligned in general; the box starts at the boundary below it (at most
// 16 - gcd(ROWB, 16) bytes earlier) and is wide enough to cover the row.
template <int KVT, int D, bool TMA>
struct DecLayout {
    static constexpr int ROWB = (D / 32) * Fmt<KVT>::BB;       // raw bytes of one head row
    static constexpr int RS = TMA ? ((ROWB + 16 - gcd16(ROWB) + 15) / 16) * 16 : ROWB;  // raw row stride in smem
    static constexpr int RAW = DT * RS;                        // raw bytes of one K (or V) tile
    static constexpr int NST = TMA ? (KVT == ARC_KV_Q8_0 ? 2 : 4) : 2;  // raw stages in flight
    static constexpr int HSTRIDE = D + 8;                      // f16 tile row stride (elements), breaks bank conflicts
    static constexpr int HBYTES = DT * HSTRIDE * 2;
    static constexpr int MERGE = WARPS * 16 * (D + 2) * 4;
    static constexpr int MAIN = NST * 2 * RAW + 2 * HBYTES;    // stages x (K,V) raw + f16 K,V
    static constexpr int BYTES = (MAIN > MERGE ? MAIN : MERGE) + 64 + 128;  // + stage barriers, alignment
    static constexpr int PIECE = (ROWB % 8 == 0) ? 8 : 4;      // cp.async granule
};

ARC_DEV void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

ARC_DEV void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

ARC_DEV void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

ARC_DEV uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
ARC_DEV __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

ARC_DEV uint32_t lds_u32(const uint8_t *p) { return *reinterpret_cast<const uint32_t *>(p); }

// Four signed bytes of w -> two half2 of the same integers (exact).
ARC_DEV void s8x4_to_h2x2(uint32_t w, __half2 &lo, __half2 &hi)
{
    const uint32_t t = w ^ 0x80808080u;
    lo = __hsub2(bits_h2(__byte_perm(t, 0x64646464u, 0x4140u)), bits_h2(0x64806480u));  // 1024 + 128
    hi = __hsub2(bits_h2(__byte_perm(t, 0x64646464u, 0x4342u)), bits_h2(0x64806480u));
}

// Four values 0..15 (one per byte of w) -> two half2 of (n - 8) (exact).
ARC_DEV void u4x4_to_h2x2(uint32_t w, __half2 &lo, __half2 &hi)
{
    lo = __hsub2(bits_h2(__byte_perm(w, 0x64646464u, 0x4140u)), bits_h2(0x64086408u));  // 1024 + 8
    hi = __hsub2(bits_h2(__byte_perm(w, 0x64646464u, 0x4342u)), bits_h2(0x64086408u));
}

// Eight bytes starting at byte offset `off` of a 4-byte-aligned row, as two words.
// Blocks are 34 or 18 bytes, so `off` is 2 mod 4 for even blocks: three aligned
// loads and a byte permute realign it without a branch.
ARC_DEV void ld8_unaligned(const uint8_t *row, int off, uint32_t &a, uint32_t &b)
{
    const uint8_t *base = row + (off & ~3);
    const uint32_t w0 = lds_u32(base), w1 = lds_u32(base + 4), w2 = lds_u32(base + 8);
    const uint32_t sel = (off & 2) ? 0x5432u : 0x3210u;
    a = __byte_perm(w0, w1, sel);
    b = __byte_perm(w1, w2, sel);
}

// Dequantise 8 consecutive elements (group grp = dims 8*grp .. 8*grp+7) of one raw
// head row into four half2 words.
template <int KVT>
ARC_DEV uint4 dequant8(const uint8_t *row, int grp)
{
    const int blk = grp >> 2, e0 = (grp & 3) * 8;
    const int boff = blk * Fmt<KVT>::BB;
    const __half2 sc = __half2half2(*reinterpret_cast<const __half *>(row + boff));
    uint32_t a, b;
    __half2 h0, h1, h2, h3;
    if constexpr (KVT == ARC_KV_Q8_0) {
        ld8_unaligned(row, boff + 2 + e0, a, b);
        s8x4_to_h2x2(a, h0, h1);
        s8x4_to_h2x2(b, h2, h3);
    } else {
        // elements 0..15 are the low nibbles of bytes 0..15, elements 16..31 the high ones
        ld8_unaligned(row, boff + 2 + (e0 & 15), a, b);
        const int sh = e0 >= 16 ? 4 : 0;
        u4x4_to_h2x2((a >> sh) & 0x0F0F0F0Fu, h0, h1);
        u4x4_to_h2x2((b >> sh) & 0x0F0F0F0Fu, h2, h3);
    }
    return make_uint4(h2_bits(__hmul2(h0, sc)), h2_bits(__hmul2(h1, sc)), h2_bits(__hmul2(h2, sc)),
                      h2_bits(__hmul2(h3, sc)));
}

template <int BYTES>
ARC_DEV void cp_async_n(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(smem_u32(dst)), "l"(src), "n"(BYTES) : "memory");
}
template <int N>
ARC_DEV void cp_async_wait_n() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int KVT, int D, bool TMA>
__global__ void __launch_bounds__(WARPS * 32) decode_split_kernel(const __grid_constant__ DecodeParams p)
{
    using L = DecLayout<KVT, D, TMA>;
    constexpr int KS = D / 16;    // k-steps of S
    constexpr int NT_O = D / 8;   // n-tiles of O

    extern __shared__ __align__(128) uint8_t smem_raw[];
    // TMA destinations 128-byte aligned (every tile size below is a multiple of 128)
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *raw = smem;                                   // [NST stages][K, V][RAW]
    __half *kh = reinterpret_cast<__half *>(smem + L::NST * 2 * L::RAW);
    __half *vh = kh + DT * L::HSTRIDE;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BYTES - 128 - 64);   // TMA stage barriers

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;

    const int s = blockIdx.x / (p.Hkv * p.splits);
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
    int row_t[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int r = g + 8 * hr;
        row_t[hr] = (r < M) ? r % sq.n_q : -1;
    }
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int pi = 0; pi < 4; ++pi) {
            const int r = g + 8 * (pi & 1);
            const int d = ks * 16 + 2 * tq + 8 * (pi >> 1);
            float2 v = make_float2(0.f, 0.f);
            if (r < M) {
                const int h = kvh * G + r / sq.n_q;
                const int tok = sq.q_begin + r % sq.n_q;
                v = *reinterpret_cast<const float2 *>(p.q + ((int64_t)tok * p.H + h) * D + d);
            }
            qa[ks][pi] = h2_bits(__floats2half2_rn(v.x * p.scale_log2, v.y * p.scale_log2));
        }
    }

    float o[NT_O][4];
#pragma unroll
    for (int i = 0; i < NT_O; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};

    const int n_tiles = c_end > c_begin ? (c_end - c_begin + DT - 1) / DT : 0;
    const uint8_t *kbase = p.k_cache + (int64_t)kvh * L::ROWB;
    const uint8_t *vbase = p.v_cache + (int64_t)kvh * L::ROWB;
    const int64_t cell_stride = (int64_t)p.Hkv * L::ROWB;
    const int pad = TMA ? (L::ROWB * kvh) & 15 : 0;       // head row offset inside a smem row
    const int x0 = L::ROWB * kvh - pad;                    // 16-byte aligned box start (bytes)

    if (TMA) {
        if (threadIdx.x == 0) {
            for (int i = 0; i < L::NST; ++i) mbar_init(&full[i], 1);
            fence_mbar_init();
        }
        __syncthreads();
    }
    // Tile i: TMA into stage i % NST (thread 0), completion on full[i % NST].
    auto issue_tma = [&](int i) {
        if (threadIdx.x == 0) {
            const int st = i % L::NST;
            uint8_t *dk = raw + st * 2 * L::RAW;
            mbar_arrive_expect_tx(&full[st], 2 * L::RAW);
            const int row = sq.kv_begin + c_begin + i * DT;
            tma_load_2d(dk, &p.tm_kc, &full[st], x0, row);
            tma_load_2d(dk + L::RAW, &p.tm_vc, &full[st], x0, row);
        }
    };
    auto issue = [&](int i) {
        uint8_t *dk = raw + (i & 1) * 2 * L::RAW;
        uint8_t *dv = dk + L::RAW;
        const int key0 = c_begin + i * DT;
        constexpr int PR = L::ROWB / L::PIECE;  // pieces per row (<= 32): one lane each
        static_assert(PR <= 32, "a head row must fit one warp instruction");
        static_assert(!TMA || L::RAW % 128 == 0, "TMA tiles keep 128-byte alignment");
        if (lane < PR) {
            const int off = lane * L::PIECE;
#pragma unroll 4
            for (int kr = warp; kr < DT; kr += WARPS) {
                const int key = min(key0 + kr, c_end - 1);  // rows past the chunk repeat a valid row; masked
                const int64_t cell = sq.kv_begin + key;
                cp_async_n<L::PIECE>(dk + kr * L::ROWB + off, kbase + cell * cell_stride + off);
                cp_async_n<L::PIECE>(dv + kr * L::ROWB + off, vbase + cell * cell_stride + off);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    if (TMA) {
        for (int i = 0; i < L::NST && i < n_tiles; ++i) issue_tma(i);
    } else {
        if (n_tiles > 0) issue(0);
        if (n_tiles > 1) issue(1);
    }
    bool ok = true;
    const uint32_t kh_s = smem_u32(kh), vh_s = smem_u32(vh);
    for (int i = 0; i < n_tiles; ++i) {
        if (TMA) {
            ok = mbar_wait(&full[i % L::NST], (uint32_t)((i / L::NST) & 1)) && ok;
        } else {
            if (i + 1 < n_tiles)
                cp_async_wait_n<1>();
            else
                cp_async_wait_n<0>();
        }
        __syncthreads();  // raw tile i visible; every warp is done with the f16 tiles of tile i-1
        {
            const uint8_t *rk = raw + (TMA ? (i % L::NST) : (i & 1)) * 2 * L::RAW + pad;
            const uint8_t *rv = rk + L::RAW;
            const int valid = c_end - (c_begin + i * DT);     // rows of this tile inside the chunk
            constexpr int GROUPS = DT * (D / 8);
#pragma unroll 2
            for (int x = threadIdx.x; x < GROUPS; x += WARPS * 32) {
                const int r = x / (D / 8), grp = x % (D / 8);  // D / 8 is a power of two
                uint4 kq = make_uint4(0, 0, 0, 0), vq = kq;
                if (!TMA || r < valid) {  // a TMA box may run past the chunk into unused cells: zeros there
                    kq = dequant8<KVT>(rk + r * L::RS, grp);
                    vq = dequant8<KVT>(rv + r * L::RS, grp);
                }
                *reinterpret_cast<uint4 *>(kh + r * L::HSTRIDE + grp * 8) = kq;
                *reinterpret_cast<uint4 *>(vh + r * L::HSTRIDE + grp * 8) = vq;
            }
        }
        __syncthreads();  // f16 tiles ready; the raw stage of tile i is free again
        if (TMA) {
            if (i + L::NST < n_tiles) issue_tma(i + L::NST);
        } else {
            if (i + 2 < n_tiles) issue(i + 2);
        }

        const int kw = warp * 16;                      // this warp's 16 keys of the tile
        const int key0 = c_begin + i * DT + kw;
        // ---- S = Q K^T, 16 rows x 16 keys (two n-tiles of 8)
        float sacc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
            const int krow = kw + nt * 8 + (lane & 7);
#pragma unroll
            for (int ks = 0; ks < KS; ks += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kh_s + (krow * L::HSTRIDE + ks * 16 + (lane >> 3) * 8) * 2, b0, b1, b2, b3);
                mma16816(sacc[nt], qa[ks], b0, b1);
                mma16816(sacc[nt], qa[ks + 1], b2, b3);
            }
        }
        // ---- mask: key index vs. the chunk end and each row's causal limit
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int lim = row_t[hr] < 0 ? -1 : sq.n_kv - sq.n_q + row_t[hr];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int key = key0 + nt * 8 + 2 * tq + e;
                    if (key >= c_end || key > lim) sacc[nt][2 * hr + e] = -INFINITY;
                }
        }
        // ---- online softmax for rows g and g+8 (a row is spread over the 4 lanes of a quad)
        uint32_t pa[4];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            float mx = fmaxf(fmaxf(sacc[0][2 * hr], sacc[0][2 * hr + 1]), fmaxf(sacc[1][2 * hr], sacc[1][2 * hr + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_r[hr], mx);
            const float msafe = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = (m_r[hr] == -INFINITY) ? 0.f : fast_exp2(m_r[hr] - msafe);
            m_r[hr] = m_new;
            const float p00 = fast_exp2(sacc[0][2 * hr] - msafe), p01 = fast_exp2(sacc[0][2 * hr + 1] - msafe);
            const float p10 = fast_exp2(sacc[1][2 * hr] - msafe), p11 = fast_exp2(sacc[1][2 * hr + 1] - msafe);
            l_r[hr] = l_r[hr] * alpha + (p00 + p01 + p10 + p11);
            if (alpha != 1.f) {
#pragma unroll
                for (int i2 = 0; i2 < NT_O; ++i2) {
                    o[i2][2 * hr] *= alpha;
                    o[i2][2 * hr + 1] *= alpha;
                }
            }
            pa[hr] = h2_bits(__floats2half2_rn(p00, p01));       // row g / g+8, keys 2tq..  (n-tile 0)
            pa[2 + hr] = h2_bits(__floats2half2_rn(p10, p11));   // keys 8 + 2tq..           (n-tile 1)
        }
        // ---- O += P V: V fragments by ldmatrix.trans from the f16 tile
        const int vrow = kw + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int nd = 0; nd < NT_O; nd += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vh_s + (vrow * L::HSTRIDE + nd * 8 + (lane >> 4) * 8) * 2, b0, b1, b2, b3);
            mma16816(o[nd], pa, b0, b1);
            mma16816(o[nd + 1], pa, b2, b3);
        }
    }

    // ---- merge the 4 warps of this CTA in shared memory
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 1);
        l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 2);
    }
    __syncthreads();
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
    if (!ok && threadIdx.x == 0) report(p.status, ST_TIMEOUT_LOAD);
    // Let the merge kernel start its prologue; it waits for this grid's writes.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Warp-specialised split kernel (TMA path).  Warp 4 streams raw K/V tiles of 64
// cells into a ring of NST stages; each of warps 0-3 owns 16 cells of every
// tile: it dequantises just those rows into its own f16 buffers, releases the
// raw stage (one arrive per warp on empty[stage]) and runs its MMAs.  No
// CTA-wide barrier inside the loop, so the four warps drift independently and
// hide one another's latencies.
constexpr int WS_WARPS = 5;

template <int KVT, int D>
struct WsLayout {
    static constexpr int ROWB = (D / 32) * Fmt<KVT>::BB;
    static constexpr int RS = ((ROWB + 16 - gcd16(ROWB) + 15) / 16) * 16;   // smem row stride of a raw tile
    static constexpr int RAW = DT * RS;
    static constexpr int NST = KVT == ARC_KV_Q8_0 ? 2 : 3;          // three CTAs per SM fit
    static constexpr int WROWS = DT / WARPS;                                  // cells per consumer warp
    static constexpr int HSTRIDE = D + 8;
    static constexpr int HW = WROWS * HSTRIDE * 2;                            // one f16 buffer (K or V) of a warp
    static constexpr int QB = 16 * HSTRIDE * 2;                               // Q tile (f16, pre-scaled)
    static constexpr int MAIN = NST * 2 * RAW + WARPS * 2 * HW + QB;
    static constexpr int MERGE = WARPS * 16 * (D + 2) * 4;
    static constexpr int BYTES = (MAIN > MERGE ? MAIN : MERGE) + 128 + 128;  // + barriers, alignment
};

// Dequantise the block that starts `off` bytes into a 16-byte-aligned raw row:
// three (q8_0) or two (q4_0) aligned 16-byte loads cover it wherever it starts,
// which with the 144 / 80-byte smem row stride touches 8 rows in distinct banks.
// `off` is a compile-time constant at every call (unrolled loops, template pad),
// so all byte positions below fold away.
template <int KVT>
ARC_DEV void dequant_block16(const uint8_t *row, int off, __half *dst)
{
    constexpr int N4 = KVT == ARC_KV_Q8_0 ? 3 : 2;
    const uint4 *w4 = reinterpret_cast<const uint4 *>(row + (off & ~15));
    const int o = off & 15;
    uint32_t W[4 * N4];
#pragma unroll
    for (int i = 0; i < N4; ++i) {
        const uint4 t = w4[i];
        W[4 * i] = t.x, W[4 * i + 1] = t.y, W[4 * i + 2] = t.z, W[4 * i + 3] = t.w;
    }
    const __half2 sc = bits_h2(__byte_perm(W[o >> 2], 0u, (o & 2) ? 0x3232u : 0x1010u));
    auto word = [&](int j) -> uint32_t {   // data bytes 4j .. 4j+3 of the block
        const int b0 = o + 2 + 4 * j;
        return (b0 & 3) ? __byte_perm(W[b0 >> 2], W[(b0 >> 2) + 1], 0x5432u) : W[b0 >> 2];
    };
    uint4 *out = reinterpret_cast<uint4 *>(dst);
    if constexpr (KVT == ARC_KV_Q8_0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __half2 h0, h1, h2, h3;
            s8x4_to_h2x2(word(2 * q), h0, h1);
            s8x4_to_h2x2(word(2 * q + 1), h2, h3);
            out[q] = make_uint4(h2_bits(__hmul2(h0, sc)), h2_bits(__hmul2(h1, sc)), h2_bits(__hmul2(h2, sc)),
                                h2_bits(__hmul2(h3, sc)));
        }
    } else {
        uint32_t d[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) d[k] = word(k);
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint32_t a = half ? (d[2 * q] >> 4) & 0x0F0F0F0Fu : d[2 * q] & 0x0F0F0F0Fu;
                const uint32_t b = half ? (d[2 * q + 1] >> 4) & 0x0F0F0F0Fu : d[2 * q + 1] & 0x0F0F0F0Fu;
                __half2 h0, h1, h2, h3;
                u4x4_to_h2x2(a, h0, h1);
                u4x4_to_h2x2(b, h2, h3);
                out[half * 2 + q] = make_uint4(h2_bits(__hmul2(h0, sc)), h2_bits(__hmul2(h1, sc)),
                                               h2_bits(__hmul2(h2, sc)), h2_bits(__hmul2(h3, sc)));
            }
    }
}

// One consumer warp's 16 rows of a raw K/V tile (kvh's head row starts PAD bytes
// into each 16-byte-aligned smem row) into its f16 buffers: at step k every lane
// takes block k, lanes 0-15 of K rows 0-15 and lanes 16-31 of V rows 0-15.
template <int KVT, int D, int PAD>
ARC_DEV void dequant_warp_rows(const uint8_t *rk, int raw_bytes, int rs, int valid, __half *kb, __half *vb, int hstride)
{
    const int lane = threadIdx.x & 31, which = lane >> 4, rr = lane & 15;
    const uint8_t *rowp = rk + which * raw_bytes + rr * rs;
    __half *dst = (which ? vb : kb) + rr * hstride;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
        if (rr < valid) {
            dequant_block16<KVT>(rowp, PAD + k * Fmt<KVT>::BB, dst + k * 32);
        } else {
            uint4 *z = reinterpret_cast<uint4 *>(dst + k * 32);
            z[0] = z[1] = z[2] = z[3] = make_uint4(0, 0, 0, 0);
        }
    }
}

template <int KVT, int D>
__global__ void __launch_bounds__(WS_WARPS * 32, 3) decode_ws_kernel(const __grid_constant__ DecodeParams p)
{
    using L = WsLayout<KVT, D>;
    constexpr int KS = D / 16;
    constexpr int NT_O = D / 8;
    constexpr int NB = D / 32;                        // blocks per row

    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *raw = smem;                                            // [NST][K, V][RAW]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BYTES - 256);
    uint64_t *empty = full + L::NST;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int s = blockIdx.x / (p.Hkv * p.splits);
    const int kvh = (blockIdx.x / p.splits) % p.Hkv;
    const int sp = blockIdx.x % p.splits;
    const arc_seq sq = p.seqs[s];
    const int G = p.H / p.Hkv;
    const int M = G * sq.n_q;
    const int c_begin = sp * p.chunk;
    const int c_end = min(c_begin + p.chunk, sq.n_kv);
    const int n_tiles = c_end > c_begin ? (c_end - c_begin + DT - 1) / DT : 0;
    const int pad = (L::ROWB * kvh) & 15;
    const int x0 = L::ROWB * kvh - pad;

    if (threadIdx.x == 0) {
        for (int i = 0; i < L::NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], WARPS);
        }
        fence_mbar_init();
    }
    __syncthreads();

    float o[NT_O][4];
#pragma unroll
    for (int i = 0; i < NT_O; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
    bool ok = true;

    if (warp == WARPS) {
        // =============================== producer
        if (lane == 0) {
            for (int i = 0; i < n_tiles && ok; ++i) {
                const int st = i % L::NST;
                if (i >= L::NST) ok = mbar_wait(&empty[st], (uint32_t)((i / L::NST - 1) & 1));
                if (!ok) break;
                uint8_t *dk = raw + st * 2 * L::RAW;
                mbar_arrive_expect_tx(&full[st], 2 * L::RAW);
                const int row = sq.kv_begin + c_begin + i * DT;
                tma_load_2d(dk, &p.tm_kc, &full[st], x0, row);
                tma_load_2d(dk + L::RAW, &p.tm_vc, &full[st], x0, row);
            }
            if (!ok) report(p.status, ST_TIMEOUT_LOAD);
        }
    } else {
        // =============================== consumer warp: 16 cells of each tile
        __half *kb = reinterpret_cast<__half *>(smem + L::NST * 2 * L::RAW + warp * 2 * L::HW);
        __half *vb = kb + L::WROWS * L::HSTRIDE;
        __half *qs = reinterpret_cast<__half *>(smem + L::NST * 2 * L::RAW + WARPS * 2 * L::HW);
        const uint32_t kb_s = smem_u32(kb), vb_s = smem_u32(vb), qs_s = smem_u32(qs);
        int row_t[2];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int r = g + 8 * hr;
            row_t[hr] = (r < M) ? r % sq.n_q : -1;
        }
        // Q tile, shared by the four warps: 16 fold rows x D, scaled into log2 units, f16.
        for (int x = threadIdx.x; x < 16 * D / 2; x += WARPS * 32) {
            const int r = x / (D / 2), d = (x % (D / 2)) * 2;
            float2 v = make_float2(0.f, 0.f);
            if (r < M) {
                const int h = kvh * G + r / sq.n_q;
                const int tok = sq.q_begin + r % sq.n_q;
                v = *reinterpret_cast<const float2 *>(p.q + ((int64_t)tok * p.H + h) * D + d);
            }
            *reinterpret_cast<__half2 *>(qs + r * L::HSTRIDE + d) = __floats2half2_rn(v.x * p.scale_log2, v.y * p.scale_log2);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32) : "memory");   // consumer warps only
        for (int i = 0; i < n_tiles; ++i) {
            const int st = i % L::NST;
            ok = mbar_wait(&full[st], (uint32_t)((i / L::NST) & 1)) && ok;
            const int kw0 = i * DT + warp * L::WROWS;              // first cell (chunk-relative) of this warp
            const int valid = c_end - c_begin - kw0;               // rows of this warp inside the chunk
            {
                const uint8_t *rk = raw + st * 2 * L::RAW + warp * L::WROWS * L::RS;   // 16-byte aligned rows
                switch (pad) {   // CTA-uniform
                case 0: dequant_warp_rows<KVT, D, 0>(rk, L::RAW, L::RS, valid, kb, vb, L::HSTRIDE); break;
                case 4: dequant_warp_rows<KVT, D, 4>(rk, L::RAW, L::RS, valid, kb, vb, L::HSTRIDE); break;
                case 8: dequant_warp_rows<KVT, D, 8>(rk, L::RAW, L::RS, valid, kb, vb, L::HSTRIDE); break;
                default: dequant_warp_rows<KVT, D, 12>(rk, L::RAW, L::RS, valid, kb, vb, L::HSTRIDE); break;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);                // this warp is done with the raw stage

            const int key0 = c_begin + kw0;
            float sacc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
                const int krow = nt * 8 + (lane & 7);
#pragma unroll
                for (int ks = 0; ks < KS; ks += 2) {
                    uint32_t b0, b1, b2, b3, qa0[4], qa1[4];
                    ldsm_x4(kb_s + (krow * L::HSTRIDE + ks * 16 + (lane >> 3) * 8) * 2, b0, b1, b2, b3);
                    ldsm_x4(qs_s + ((lane & 15) * L::HSTRIDE + ks * 16 + (lane >> 4) * 8) * 2, qa0[0], qa0[1], qa0[2],
                            qa0[3]);
                    ldsm_x4(qs_s + ((lane & 15) * L::HSTRIDE + (ks + 1) * 16 + (lane >> 4) * 8) * 2, qa1[0], qa1[1],
                            qa1[2], qa1[3]);
                    mma16816(sacc[nt], qa0, b0, b1);
                    mma16816(sacc[nt], qa1, b2, b3);
                }
            }
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int lim = row_t[hr] < 0 ? -1 : sq.n_kv - sq.n_q + row_t[hr];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int key = key0 + nt * 8 + 2 * tq + e;
                        if (key >= c_end || key > lim) sacc[nt][2 * hr + e] = -INFINITY;
                    }
            }
            uint32_t pa[4];
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                float mx = fmaxf(fmaxf(sacc[0][2 * hr], sacc[0][2 * hr + 1]), fmaxf(sacc[1][2 * hr], sacc[1][2 * hr + 1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m_r[hr], mx);
                const float msafe = (m_new == -INFINITY) ? 0.f : m_new;
                const float alpha = (m_r[hr] == -INFINITY) ? 0.f : fast_exp2(m_r[hr] - msafe);
                m_r[hr] = m_new;
                const float p00 = fast_exp2(sacc[0][2 * hr] - msafe), p01 = fast_exp2(sacc[0][2 * hr + 1] - msafe);
                const float p10 = fast_exp2(sacc[1][2 * hr] - msafe), p11 = fast_exp2(sacc[1][2 * hr + 1] - msafe);
                l_r[hr] = l_r[hr] * alpha + (p00 + p01 + p10 + p11);
                if (alpha != 1.f) {
#pragma unroll
                    for (int i2 = 0; i2 < NT_O; ++i2) {
                        o[i2][2 * hr] *= alpha;
                        o[i2][2 * hr + 1] *= alpha;
                    }
                }
                pa[hr] = h2_bits(__floats2half2_rn(p00, p01));
                pa[2 + hr] = h2_bits(__floats2half2_rn(p10, p11));
            }
            const int vrow = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int nd = 0; nd < NT_O; nd += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vb_s + (vrow * L::HSTRIDE + nd * 8 + (lane >> 4) * 8) * 2, b0, b1, b2, b3);
                mma16816(o[nd], pa, b0, b1);
                mma16816(o[nd + 1], pa, b2, b3);
            }
            __syncwarp();   // every lane's ldmatrix of this warp's buffers is done before the next dequant
        }
        if (!ok && lane == 0) report(p.status, ST_TIMEOUT_LOAD);
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 1);
            l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 2);
        }
    }

    // ---- merge the 4 consumer warps (the raw ring and f16 buffers are idle now)
    __syncthreads();
    float *so = reinterpret_cast<float *>(smem);
    float *sml = so + WARPS * 16 * D;
    if (warp < WARPS) {
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
    }
    __syncthreads();
    const int64_t part = (int64_t)blockIdx.x;
    for (int x = threadIdx.x; x < 16 * D; x += WS_WARPS * 32) {
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
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Merge the chunk partials of one (sequence, kv head, fold row) by their
// log-sum-exp weights, normalise, write O and LSE.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const __grid_constant__ DecodeParams p)
{
    __shared__ float s_w[256];     // per-split weight exp2(m_sp - m)
    __shared__ float s_red[2];
    const int s = blockIdx.x / p.Hkv, kvh = blockIdx.x % p.Hkv, r = blockIdx.y;
    const arc_seq sq = p.seqs[s];
    const int G = p.H / p.Hkv;
    if (r >= G * sq.n_q) return;
    const int h = kvh * G + r / sq.n_q, tok = sq.q_begin + r % sq.n_q;
    const int d = threadIdx.x;
    const int64_t part0 = ((int64_t)s * p.Hkv + kvh) * p.splits;
    asm volatile("griddepcontrol.wait;" ::: "memory");  // partials of the split kernel are complete
    if (d == 0) {
        float mm = -INFINITY;
        for (int sp = 0; sp < p.splits; ++sp) mm = fmaxf(mm, p.ws_ml[((part0 + sp) * 16 + r) * 2]);
        const float ms = (mm == -INFINITY) ? 0.f : mm;
        float ll = 0.f;
        for (int sp = 0; sp < p.splits; ++sp) {
            const float mw = p.ws_ml[((part0 + sp) * 16 + r) * 2];
            const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - ms);
            s_w[sp] = f;
            ll += f * p.ws_ml[((part0 + sp) * 16 + r) * 2 + 1];
        }
        s_red[0] = mm;
        s_red[1] = ll;
    }
    __syncthreads();
    const float mm = s_red[0], ll = s_red[1];
    float acc = 0.f;
#pragma unroll 4
    for (int sp = 0; sp < p.splits; ++sp) acc += s_w[sp] * p.ws_o[((part0 + sp) * 16 + r) * D + d];
    p.o[((int64_t)tok * p.H + h) * D + d] = ll > 0.f ? acc / ll : 0.f;
    if (d == 0) p.lse[(int64_t)tok * p.H + h] = ll > 0.f ? (mm + log2f(ll)) * LN2 : -INFINITY;
}

template <int KVT, int D, bool TMA>
cudaError_t launch_t(const DecodeParams &p, cudaStream_t s)
{
    const int grid = p.n_seq * p.Hkv * p.splits;
    if (grid == 0) return cudaSuccess;
    cudaError_t e;
    if (TMA) {
        auto k1 = decode_ws_kernel<KVT, D>;
        const int bytes = WsLayout<KVT, D>::BYTES;
        if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess) return e;
        k1<<<grid, WS_WARPS * 32, bytes, s>>>(p);
    } else {
        auto k1 = decode_split_kernel<KVT, D, false>;
        const int bytes = DecLayout<KVT, D, false>::BYTES;
        if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess) return e;
        k1<<<grid, WARPS * 32, bytes, s>>>(p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // The merge launches as a programmatic dependent: its launch overlaps the
    // split kernel's tail and it waits (griddepcontrol.wait) for the partials.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_seq * p.Hkv, 16);
    cfg.blockDim = dim3(D);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, p);
}

template <bool TMA>
int smem_t(int kv_type, int D)
{
    if (TMA) {
        if (kv_type == ARC_KV_Q8_0) return D == 64 ? WsLayout<ARC_KV_Q8_0, 64>::BYTES : WsLayout<ARC_KV_Q8_0, 128>::BYTES;
        return D == 64 ? WsLayout<ARC_KV_Q4_0, 64>::BYTES : WsLayout<ARC_KV_Q4_0, 128>::BYTES;
    }
    if (kv_type == ARC_KV_Q8_0)
        return D == 64 ? DecLayout<ARC_KV_Q8_0, 64, false>::BYTES : DecLayout<ARC_KV_Q8_0, 128, false>::BYTES;
    return D == 64 ? DecLayout<ARC_KV_Q4_0, 64, false>::BYTES : DecLayout<ARC_KV_Q4_0, 128, false>::BYTES;
}

template <bool TMA>
cudaError_t launch_k(const DecodeParams &p, cudaStream_t s)
{
    if (p.kv_type == ARC_KV_Q8_0) {
        if (p.D == 64) return launch_t<ARC_KV_Q8_0, 64, TMA>(p, s);
        if (p.D == 128) return launch_t<ARC_KV_Q8_0, 128, TMA>(p, s);
    } else {
        if (p.D == 64) return launch_t<ARC_KV_Q4_0, 64, TMA>(p, s);
        if (p.D == 128) return launch_t<ARC_KV_Q4_0, 128, TMA>(p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

int decode_smem_bytes(int kv_type, int D, bool tma) { return tma ? smem_t<true>(kv_type, D) : smem_t<false>(kv_type, D); }

// Box width in bytes of the TMA path (covers a head row from the 16-byte boundary below it).
int decode_box_bytes(int kv_type, int D)
{
    if (kv_type == ARC_KV_Q8_0) return D == 64 ? DecLayout<ARC_KV_Q8_0, 64, true>::RS : DecLayout<ARC_KV_Q8_0, 128, true>::RS;
    return D == 64 ? DecLayout<ARC_KV_Q4_0, 64, true>::RS : DecLayout<ARC_KV_Q4_0, 128, true>::RS;
}

cudaError_t launch_decode(const DecodeParams &p, cudaStream_t s)
{
    if (p.splits > 256) return cudaErrorInvalidValue;
    return p.tma ? launch_k<true>(p, s) : launch_k<false>(p, s);
}

}  // namespace arc
