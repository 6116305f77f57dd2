// decode.cu -- multi-sequence decode over a unified q8_0 / q4_0 KV cache.
//
// The quantised K/V blocks are never converted as a whole: each CTA copies the
// raw bytes of a 64-key tile into shared memory and dequantises them right
// before the tensor cores use them ("unsloth llama.cpp: dequantize q4_0/q8_0
// K/V tiles in the FA MMA kernel", summary: tiles are dequantised as they are
// loaded instead of a whole-cache f16 conversion per layer per step).  Each
// element is dequantised exactly once.  Two kernels do this:
//   decode_ws_kernel (TMA path, cache rows at 16-byte multiples): a producer
//     warp streams raw tiles by TMA; the consumer warps build their mma.sync
//     operands in registers straight from the raw bytes (no f16 tile in shared
//     memory), in a dim order matched to the block layout.
//   decode_split_kernel (any cell stride): cp.async copies, one cooperative
//     pass into an f16 tile, ldmatrix (K) and ldmatrix.trans (V) fragments.
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

#include <type_traits>

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

// Shared memory of the in-CTA merge of the WARPS consumer warps: per-warp O
// partials with a padded row stride (D + 8 floats: the fragment stores of the 8
// row groups of a warp land in distinct banks), per-warp row max / sum, the
// merge weights and the merged row max / sum.
template <int D>
struct MergeLayout {
    static constexpr int OS = D + 8;
    static constexpr int BYTES = (WARPS * 16 * OS + WARPS * 16 * 2 + WARPS * 16 + 16 * 2) * 4;
};

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
    static constexpr int MERGE = MergeLayout<D>::BYTES;
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

// Merge the consumer warps of this CTA (each holding an online-softmax partial of
// 16 fold rows: unnormalised O fragments, row max, row sum) into the CTA's one
// partial in the workspace, weighting each warp by exp2(m_warp - m) as in the
// log-sum-exp merge of split attention.  Called by all NTHR threads of the CTA
// after the main loop; `consumer` marks the threads that hold fragments.
//
// PERM = false: fragment n-tile nd, column c holds dim 8*nd + c (the plain
// m16n8k16 layout).  PERM = true: the B operand of P V was loaded with a
// permuted dim order (lane group g takes the D/8 consecutive dims D/8*g ...), so
// column c of n-tile nd holds dim D/8*c + nd.  In shared memory dim d then sits
// at column d + 2*(d / (D/4)): the skew spreads the four lanes of a quad, whose
// dims are D/4 apart, over different banks.
template <int D, int NTHR, bool PERM>
ARC_DEV void write_cta_partial(const float (&o)[D / 8][4], const float (&m_r)[2], const float (&l_r)[2], bool consumer,
                               uint8_t *smem, const DecodeParams &p, int64_t part)
{
    using ML = MergeLayout<D>;
    constexpr int ND = D / 8;
    float *so = reinterpret_cast<float *>(smem);        // [WARPS][16][OS]
    float *sml = so + WARPS * 16 * ML::OS;              // [WARPS][16][2]
    float *swt = sml + WARPS * 16 * 2;                  // [WARPS][16]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    __syncthreads();   // every warp is past its last read of the tile buffers this overlays
    if (consumer) {
#pragma unroll
        for (int nd = 0; nd < ND; ++nd)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                float *row = so + (warp * 16 + g + 8 * hr) * ML::OS;
                if constexpr (PERM) {
                    // dims 2*ND*tq + nd and 2*ND*tq + ND + nd, skewed by 2*tq
                    row[2 * ND * tq + nd + 2 * tq] = o[nd][2 * hr];
                    row[2 * ND * tq + ND + nd + 2 * tq] = o[nd][2 * hr + 1];
                } else {
                    *reinterpret_cast<float2 *>(row + nd * 8 + 2 * tq) = make_float2(o[nd][2 * hr], o[nd][2 * hr + 1]);
                }
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
    if (threadIdx.x < 16) {
        const int r = threadIdx.x;
        float mm = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) mm = fmaxf(mm, sml[(w * 16 + r) * 2]);
        const float ms = (mm == -INFINITY) ? 0.f : mm;
        float ll = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float mw = sml[(w * 16 + r) * 2];
            const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - ms);
            swt[w * 16 + r] = f;
            ll += f * sml[(w * 16 + r) * 2 + 1];
        }
        *reinterpret_cast<float2 *>(p.ws_ml + (part * 16 + r) * 2) = make_float2(mm, ll);
    }
    __syncthreads();
    if constexpr (PERM) {
        constexpr int D2 = D / 2;
#pragma unroll
        for (int x = threadIdx.x; x < 16 * D2; x += NTHR) {
            const int r = x / D2, d = (x % D2) * 2;
            const int col = d + 2 * (d / (D / 4));
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int w = 0; w < WARPS; ++w) {
                const float f = swt[w * 16 + r];
                const float2 v = *reinterpret_cast<const float2 *>(so + (w * 16 + r) * ML::OS + col);
                acc.x += f * v.x, acc.y += f * v.y;
            }
            *reinterpret_cast<float2 *>(p.ws_o + (part * 16 + r) * D + d) = acc;
        }
    } else {
        constexpr int D4 = D / 4;
#pragma unroll
        for (int x = threadIdx.x; x < 16 * D4; x += NTHR) {
            const int r = x / D4, d = (x % D4) * 4;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < WARPS; ++w) {
                const float f = swt[w * 16 + r];
                const float4 v = *reinterpret_cast<const float4 *>(so + (w * 16 + r) * ML::OS + d);
                acc.x += f * v.x, acc.y += f * v.y, acc.z += f * v.z, acc.w += f * v.w;
            }
            *reinterpret_cast<float4 *>(p.ws_o + (part * 16 + r) * D + d) = acc;
        }
    }
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
    uint8_t *smem = align_smem<128>(smem_raw);
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
    write_cta_partial<D, WARPS * 32, false>(o, m_r, l_r, true, smem, p, part);
    if (!ok && threadIdx.x == 0) report(p.status, ST_TIMEOUT_LOAD);
    // Let the merge kernel start its prologue; it waits for this grid's writes.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}


// ---------------------------------------------------------------------------
// Warp-specialised split kernel (TMA path).  Warp 4 streams raw K/V tiles into
// a ring of NST stages; warps 0-3 build their mma.sync operands straight from
// the raw bytes, in registers: no f16 copy of a tile is ever written, so shared
// memory carries only the TMA writes, one read of each raw byte and Q.
//
// Shapes.  A CTA takes ROWS = 16*MF fold rows (MF m16 fragments) of one
// (sequence, kv head, row group, chunk).  The head dim is cut into NS slices of
// KS = D/NS dims, so that one warp's O accumulators (MF x KS/2 floats a lane)
// stay at or under 64 registers; the 4 consumer warps are NCG = 4/NS cell
// groups x NS slices, and a tile holds DT = 16*NCG cells.  Warp (cg, s) owns the
// 16 cells cg*16.. of every tile and the dims of slice s, for K as for V:
//   S  = Q K^T: the warp's partial over its slice's dims; the NS partials of a
//        cell group are summed through shared memory in slice order, so every
//        warp of the group holds the same S and runs the same online softmax;
//   O += P V:   the warp's slice of the output dims.
// Every raw byte is dequantised once.  With NS = 1 (D <= 128, MF = 1; the
// multi-sequence decode) there is no exchange and a tile has 64 cells.
//
// Dim permutations.  A dot product does not change when the same permutation
// is applied to the head dim of both operands, so S = Q K^T takes the k-step
// order that suits the q8_0 / q4_0 block layout: in k-step j (block b = j/2,
// half hh = j%2) the lane with quad index t holds the four consecutive dims
// 32b + 16hh + 4t .. +3 (k positions 2t, 2t+1, 2t+8, 2t+9 of the fragment).
// Those are four consecutive bytes of one block (q8_0), or the low / high
// nibbles of four consecutive bytes (q4_0), so each B fragment register pair
// comes from one 32-bit word; the Q fragments are read from shared memory in
// the same order.  For O += P V the n index is the output dim: lane group g
// loads slice dims KS/8*g .. KS/8*g + KS/8 - 1 (consecutive bytes again, inside
// one block) and n-tile nd column c accumulates slice dim KS/8*c + nd, which the
// in-CTA merge undoes.
constexpr int WS_WARPS = 5;

template <int D, int MF>
struct WsShape {
    static constexpr int NS = (D * MF) / 128 < 1 ? 1 : (D * MF) / 128;   // dim slices
    static constexpr int NCG = 4 / NS;                                      // cell groups
    static constexpr int KS = D / NS;                                       // dims per slice
    static constexpr int DT = 16 * NCG;                                     // cells per tile
    static constexpr int ROWS = 16 * MF;                                    // fold rows per CTA
    static_assert(NS * NCG == 4 && KS % 32 == 0, "four consumer warps over whole blocks");
    static_assert(MF * KS <= 128, "O accumulators of a warp stay within 64 registers");
};

template <int KVT, int D, int MF>
struct WsLayout {
    using S = WsShape<D, MF>;
    static constexpr int BB = Fmt<KVT>::BB;
    static constexpr int ROWB = (D / 32) * BB;                              // raw bytes of a head row
    static constexpr int SB = (S::KS / 32) * BB;                            // raw bytes of one slice of it
    // smem row stride of a slice box: the box starts at the 16-byte boundary at or
    // below the slice (at most 16 - gcd(SB, 16) bytes earlier) and covers it
    static constexpr int RS = ((SB + 16 - gcd16(SB) + 15) / 16) * 16;
    static constexpr int SLICE = S::DT * RS;                                // one K (or V) slice box
    static constexpr int STAGE = S::NS * 2 * SLICE;                         // [slice][K, V] of one tile
    static constexpr int NST = STAGE >= 16384 ? 3 : 4;                      // stages in flight; three CTAs per SM fit
    // Q tile (f16, pre-scaled), stored as the m16n8k16 A fragments themselves: one 16-byte
    // record per (fragment, k-step, row group g, quad index t), so a lane's operand quad
    // is one shared load (no register moves to assemble it)
    static constexpr int QB = S::ROWS * D * 2;
    static constexpr int XB = S::NS > 1 ? 2 * S::NCG * S::NS * MF * 32 * 8 * 4 : 0;   // S partials, 2 buffers
    static constexpr int MAIN = NST * STAGE + QB + XB;
    // in-CTA merge: per cell group O [ROWS][OS] with OS = D + 8*NS (a skew of up to 6
    // floats per slice), row (max, sum), weights; merged (max, sum)
    static constexpr int OS = D + 8 * S::NS;
    static constexpr int MERGE = (S::NCG * S::ROWS * OS + S::NCG * S::ROWS * 3 + S::ROWS * 2) * 4;
    static constexpr int BYTES = (MAIN > MERGE ? MAIN : MERGE) + 128 + 128;  // + barriers, alignment
    static_assert(RS <= 256, "one TMA box per slice row");
    static_assert(ROWB % 4 == 0 && SB % 4 == 0, "slice rows start 4-byte aligned in shared memory");
    static_assert(STAGE % 128 == 0 && SLICE % 128 == 0, "TMA destinations stay 128-byte aligned");
};

ARC_DEV uint2 lds_u64(const void *p) { return *reinterpret_cast<const uint2 *>(p); }

// The 32-bit word of a raw row at byte offset OFF (OFF % 4 is 0 or 2; the row
// pointer is 4-byte aligned).
template <int OFF>
ARC_DEV uint32_t raw_word(const uint8_t *row)
{
    if constexpr ((OFF & 3) == 0) {
        return lds_u32(row + OFF);
    } else {
        return __byte_perm(lds_u32(row + (OFF & ~3)), lds_u32(row + (OFF & ~3) + 4), 0x5432u);
    }
}

// The scale of block B of a raw row, replicated into both halves of a half2.
template <int KVT, int B>
ARC_DEV __half2 raw_scale(const uint8_t *row)
{
    constexpr int OFF = B * Fmt<KVT>::BB;
    return bits_h2(__byte_perm(lds_u32(row + (OFF & ~3)), 0u, (OFF & 2) ? 0x3232u : 0x1010u));
}

// The B fragments of K block B (of the slice row `row`) for the lane with quad index
// t: kf[hh] = {b0, b1} of k-step 2B + hh (dims 32B + 16hh + 4t .. +3 of this cell).
template <int KVT, int B>
ARC_DEV void k_block_frags(const uint8_t *row, int t, uint32_t (&kf)[2][2])
{
    const __half2 sc = raw_scale<KVT, B>(row);
    const uint8_t *rt = row + 4 * t;
    __half2 lo, hi;
    if constexpr (KVT == ARC_KV_Q8_0) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            s8x4_to_h2x2(hh ? raw_word<B * 34 + 2 + 16>(rt) : raw_word<B * 34 + 2>(rt), lo, hi);
            kf[hh][0] = h2_bits(__hmul2(lo, sc));
            kf[hh][1] = h2_bits(__hmul2(hi, sc));
        }
    } else {
        const uint32_t w = raw_word<B * 18 + 2>(rt);     // low nibbles: dims +0..3, high nibbles: dims +16..19
        u4x4_to_h2x2(w & 0x0F0F0F0Fu, lo, hi);
        kf[0][0] = h2_bits(__hmul2(lo, sc));
        kf[0][1] = h2_bits(__hmul2(hi, sc));
        u4x4_to_h2x2((w >> 4) & 0x0F0F0F0Fu, lo, hi);
        kf[1][0] = h2_bits(__hmul2(lo, sc));
        kf[1][1] = h2_bits(__hmul2(hi, sc));
    }
}

// One V cell as this lane needs it: the KS/8 slice dims starting at KS/8*g (NW data
// words, realigned) and the word holding that block's scale (0 past the end of the
// chunk, which zeroes the cell: its data bytes are finite integers).
template <int KVT, int KS>
struct VCell {
    static constexpr int NW = KS / 32;   // KS/8 bytes (q8_0) or nibbles in KS/8 bytes' halves (q4_0), as words
    uint32_t d[NW];
    uint32_t sw;
};

template <int KVT, int KS>
ARC_DEV void load_vcell(const uint8_t *row, int vbase, uint32_t vsel, int soff4, bool valid, VCell<KVT, KS> &c)
{
    const uint8_t *b = row + vbase;
    uint32_t w[VCell<KVT, KS>::NW + 1];
#pragma unroll
    for (int i = 0; i <= VCell<KVT, KS>::NW; ++i) w[i] = lds_u32(b + 4 * i);
#pragma unroll
    for (int i = 0; i < VCell<KVT, KS>::NW; ++i) c.d[i] = __byte_perm(w[i], w[i + 1], vsel);
    c.sw = valid ? lds_u32(row + soff4) : 0u;
}

// The decode workspace (and the combine kernel's view of it): partial results of
// part = ((sequence * Hkv + kv head) * row_groups + row group) * splits + split,
// ROWS = 16*MF fold rows each: O [part][ROWS][D] (unnormalised) and (max, sum)
// [part][ROWS][2], in log2 units.
ARC_DEV int64_t part_index(const DecodeParams &p, int s, int kvh, int rg, int sp)
{
    return (((int64_t)s * p.Hkv + kvh) * p.row_groups + rg) * p.splits + sp;
}

// Merge the 4 consumer warps of a CTA into its one partial in the workspace: O of
// cell group cg is weighted by exp2(m_cg - m) (the log-sum-exp merge of split
// attention), slices are placed side by side.  Called by all threads of the CTA
// after the main loop; the raw ring is idle by then and is overlaid.
template <int KVT, int D, int MF>
ARC_DEV void write_ws_partial(const float (&o)[MF][WsShape<D, MF>::KS / 8][4], const float (&m_r)[MF][2],
                              const float (&l_r)[MF][2], int cg, int s, bool consumer, uint8_t *smem,
                              const DecodeParams &p, int64_t part)
{
    using SH = WsShape<D, MF>;
    using L = WsLayout<KVT, D, MF>;
    constexpr int ND = SH::KS / 8, ROWS = SH::ROWS, NCG = SH::NCG, KS = SH::KS;
    float *so = reinterpret_cast<float *>(smem);              // [NCG][ROWS][OS]
    float *sml = so + NCG * ROWS * L::OS;                     // [NCG][ROWS][2]
    float *swt = sml + NCG * ROWS * 2;                        // [NCG][ROWS]
    const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    __syncthreads();   // every warp is past its last read of the ring this overlays
    if (consumer) {
        float *base = so + cg * ROWS * L::OS + s * (KS + 8);
#pragma unroll
        for (int f = 0; f < MF; ++f)
#pragma unroll
            for (int nd = 0; nd < ND; ++nd)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    // slice dims 2*ND*tq + nd and 2*ND*tq + ND + nd, skewed by 2*tq
                    float *row = base + (f * 16 + g + 8 * hr) * L::OS;
                    row[2 * ND * tq + nd + 2 * tq] = o[f][nd][2 * hr];
                    row[2 * ND * tq + ND + nd + 2 * tq] = o[f][nd][2 * hr + 1];
                }
        if (s == 0 && tq == 0) {
#pragma unroll
            for (int f = 0; f < MF; ++f)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int r = f * 16 + g + 8 * hr;
                    sml[(cg * ROWS + r) * 2 + 0] = m_r[f][hr];
                    sml[(cg * ROWS + r) * 2 + 1] = l_r[f][hr];
                }
        }
    }
    __syncthreads();
    if (threadIdx.x < ROWS) {
        const int r = threadIdx.x;
        float mm = -INFINITY;
#pragma unroll
        for (int c = 0; c < NCG; ++c) mm = fmaxf(mm, sml[(c * ROWS + r) * 2]);
        const float ms = (mm == -INFINITY) ? 0.f : mm;
        float ll = 0.f;
#pragma unroll
        for (int c = 0; c < NCG; ++c) {
            const float mw = sml[(c * ROWS + r) * 2];
            const float w = (mw == -INFINITY) ? 0.f : fast_exp2(mw - ms);
            swt[c * ROWS + r] = w;
            ll += w * sml[(c * ROWS + r) * 2 + 1];
        }
        *reinterpret_cast<float2 *>(p.ws_ml + (part * ROWS + r) * 2) = make_float2(mm, ll);
    }
    __syncthreads();
    constexpr int D2 = D / 2;
    for (int x = threadIdx.x; x < ROWS * D2; x += WS_WARPS * 32) {
        const int r = x / D2, d = (x % D2) * 2;
        const int sl = d / KS, dd = d % KS;
        const int col = sl * (KS + 8) + dd + 2 * (dd / (KS / 4));
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < NCG; ++c) {
            const float w = swt[c * ROWS + r];
            const float2 v = *reinterpret_cast<const float2 *>(so + (c * ROWS + r) * L::OS + col);
            acc.x += w * v.x, acc.y += w * v.y;
        }
        *reinterpret_cast<float2 *>(p.ws_o + (part * ROWS + r) * D + d) = acc;
    }
}

// Three CTAs per SM with one fragment; with two, the second fragment's S and O
// registers need the room of two CTAs per SM.
template <int KVT, int D, int MF>
__global__ void __launch_bounds__(WS_WARPS * 32, MF == 1 ? 3 : 2) decode_ws_kernel(const __grid_constant__ DecodeParams p)
{
    using SH = WsShape<D, MF>;
    using L = WsLayout<KVT, D, MF>;
    constexpr int NS = SH::NS, NCG = SH::NCG, KS = SH::KS, DT = SH::DT, ROWS = SH::ROWS;
    constexpr int NB = KS / 32;                       // blocks per slice
    constexpr int ND = KS / 8;                        // P V n-tiles = slice dims per lane group
    constexpr int NW = VCell<KVT, KS>::NW;

    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *smem = align_smem<128>(smem_raw);
    uint8_t *raw = smem;                                            // [NST][NS][K, V][SLICE]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BYTES - 256);
    uint64_t *empty = full + L::NST;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int s_idx = blockIdx.x / (p.Hkv * p.row_groups * p.splits);
    const int kvh = (blockIdx.x / (p.row_groups * p.splits)) % p.Hkv;
    const int rg = (blockIdx.x / p.splits) % p.row_groups;
    const int sp = blockIdx.x % p.splits;
    const arc_seq sq = p.seqs[s_idx];
    const int G = p.H / p.Hkv;
    const int M = G * sq.n_q;
    const int r0 = rg * ROWS;                     // first fold row of this CTA
    if (r0 >= M) return;                          // a row group this sequence does not have (uniform)
    const int c_begin = sp * p.chunk;
    const int c_end = min(c_begin + p.chunk, sq.n_kv);
    const int n_tiles = c_end > c_begin ? (c_end - c_begin + DT - 1) / DT : 0;

    // Q tile: ROWS fold rows x D fp32, QI float2 per consumer thread.  The first QP
    // loads go out before anything waits (up to 8 a thread, so large tiles do not
    // hold registers the accumulators need); the rest follow the barrier below.
    constexpr int QI = ROWS * D / 2 / (4 * 32);
    constexpr int QP = QI < 8 ? QI : 8;
    static_assert(QI * 4 * 32 == ROWS * D / 2, "Q tile split");
    auto q_load = [&](int j) {
        const int x = threadIdx.x + j * 4 * 32;
        const int r = x / (D / 2), d = (x % (D / 2)) * 2;
        float2 v = make_float2(0.f, 0.f);
        if (warp < 4 && r0 + r < M) {
            const int h = kvh * G + (r0 + r) / sq.n_q;
            const int tok = sq.q_begin + (r0 + r) % sq.n_q;
            v = __ldg(reinterpret_cast<const float2 *>(p.q + ((int64_t)tok * p.H + h) * D + d));
        }
        return v;
    };
    float2 qv[QP];
#pragma unroll
    for (int j = 0; j < QP; ++j) qv[j] = q_load(j);

    float o[MF][ND][4];
#pragma unroll
    for (int f = 0; f < MF; ++f)
#pragma unroll
        for (int i = 0; i < ND; ++i) o[f][i][0] = o[f][i][1] = o[f][i][2] = o[f][i][3] = 0.f;
    float m_r[MF][2], l_r[MF][2];
#pragma unroll
    for (int f = 0; f < MF; ++f) m_r[f][0] = m_r[f][1] = -INFINITY, l_r[f][0] = l_r[f][1] = 0.f;
    bool ok = true;
    const int s = warp % NS, cg = warp / NS;       // this consumer warp's dim slice and cell group

    if (warp == 4) {
        // =============================== producer
        // It initialises the stage barriers itself and only signals the consumers
        // (bar.arrive), so its first loads go out without waiting for the Q tile.
        if (lane == 0) {
            for (int i = 0; i < L::NST; ++i) {
                mbar_init(&full[i], 1);
                mbar_init(&empty[i], 4);
            }
            fence_mbar_init();
        }
        __syncwarp();
        asm volatile("bar.arrive 2, %0;" ::"n"(WS_WARPS * 32) : "memory");
        if (lane == 0) {
            for (int i = 0; i < n_tiles && ok; ++i) {
                const int st = i % L::NST;
                if (i >= L::NST) ok = mbar_wait_sleep(&empty[st], (uint32_t)((i / L::NST - 1) & 1));
                if (!ok) break;
                uint8_t *dk = raw + st * L::STAGE;
                mbar_arrive_expect_tx(&full[st], L::STAGE);
                const int row = sq.kv_begin + c_begin + i * DT;
#pragma unroll
                for (int sl = 0; sl < NS; ++sl) {
                    const int off = L::ROWB * kvh + L::SB * sl;
                    const int x0 = off - (off & 15);
                    tma_load_2d(dk + sl * 2 * L::SLICE, &p.tm_kc, &full[st], x0, row);
                    tma_load_2d(dk + sl * 2 * L::SLICE + L::SLICE, &p.tm_vc, &full[st], x0, row);
                }
            }
            if (!ok) report(p.status, ST_TIMEOUT_LOAD);
        }
    } else {
        // =============================== consumer warp (cg, s): 16 cells of each tile, slice s
        __half *qs = reinterpret_cast<__half *>(smem + L::NST * L::STAGE);
        float4 *xbuf = reinterpret_cast<float4 *>(smem + L::NST * L::STAGE + L::QB);   // [2][NCG][NS][MF][2][32]
        int row_t[MF][2];
#pragma unroll
        for (int f = 0; f < MF; ++f)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = r0 + f * 16 + g + 8 * hr;
                row_t[f][hr] = (r < M) ? r % sq.n_q : -1;
            }
        // slice row offset inside its box row: a multiple of 4 (ROWB and SB are), so the
        // row pointers below stay 4-byte aligned and each offset keeps its own alignment
        const int pad = (L::ROWB * kvh + L::SB * s) & 15;
        // This lane's V dims KS/8*g .. of the slice: block vb, first element ve of that
        // block.  Offsets are from the slice row's first byte.
        const int vb = (ND * g) / 32, ve = (ND * g) % 32;
        const int voff = vb * L::BB + 2 + (KVT == ARC_KV_Q8_0 ? ve : (ve & 15));   // first data byte
        const int vbase = voff & ~3;
        const uint32_t vsel = (voff & 2) ? 0x5432u : 0x3210u;
        const int soff = vb * L::BB;                                              // the block's scale
        const int soff4 = soff & ~3;
        const uint32_t spair = (soff & 2) ? 0x7632u : 0x5410u;     // {scale of cell A, scale of cell B}
        const int vsh = (KVT == ARC_KV_Q4_0 && ve >= 16) ? 4 : 0;  // q4_0: high nibbles hold elements 16..31

        asm volatile("bar.sync 2, %0;" ::"n"(WS_WARPS * 32) : "memory");   // stage barriers initialised
        // Q tile, shared by the four warps: ROWS fold rows x D, scaled into log2 units, f16,
        // written as A fragments.  In k-step ks the lane with quad index t holds dims
        // 16 ks + 4t .. +3 (the permuted k order below): record (f, ks, g, t) is
        // {rows g, g+8} x {dims +0..1, +2..3}, as a0 = (g, +0..1), a1 = (g+8, +0..1),
        // a2 = (g, +2..3), a3 = (g+8, +2..3).
        uint32_t *qw = reinterpret_cast<uint32_t *>(qs);
#pragma unroll
        for (int j = 0; j < QI; ++j) {
            const int x = threadIdx.x + j * 4 * 32;
            const int r = x / (D / 2), d = (x % (D / 2)) * 2;
            const float2 v = j < QP ? qv[j < QP ? j : 0] : q_load(j);
            const int f = r / 16, gg = r % 8, up = (r % 16) / 8;
            const int ks = d / 16, t = (d % 16) / 4, hi = (d % 4) / 2;
            qw[(((f * (D / 16) + ks) * 8 + gg) * 4 + t) * 4 + hi * 2 + up] =
                h2_bits(__floats2half2_rn(v.x * p.scale_log2, v.y * p.scale_log2));
        }
        asm volatile("bar.sync 1, %0;" ::"n"(4 * 32) : "memory");   // consumer warps only
        const uint4 *qfrag = reinterpret_cast<const uint4 *>(qs) + ((s * (KS / 16)) * 8 + g) * 4 + tq;

        for (int i = 0; i < n_tiles; ++i) {
            const int st = i % L::NST;
            ok = mbar_wait(&full[st], (uint32_t)((i / L::NST) & 1)) && ok;
            const int kw0 = i * DT + cg * 16;                      // first cell (chunk-relative) of this warp
            const int valid = c_end - c_begin - kw0;               // cells of this warp inside the chunk
            const uint8_t *kt = raw + st * L::STAGE + s * 2 * L::SLICE + cg * 16 * L::RS + pad;   // this warp's 16 K rows
            const uint8_t *vt = kt + L::SLICE;

            // ---- V words for cells 2t, 2t+1, 2t+8, 2t+9 (loaded early; used after the softmax)
            VCell<KVT, KS> vc[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int cell = 2 * tq + (c & 1) + 8 * (c >> 1);
                load_vcell<KVT, KS>(vt + cell * L::RS, vbase, vsel, soff4, cell < valid, vc[c]);
            }

            // ---- S = Q K^T over the permuted k order of this slice; cells g and g+8
            float sacc[MF][2][4];
#pragma unroll
            for (int f = 0; f < MF; ++f)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) sacc[f][nt][0] = sacc[f][nt][1] = sacc[f][nt][2] = sacc[f][nt][3] = 0.f;
            const uint8_t *k0 = kt + g * L::RS, *k1 = k0 + 8 * L::RS;
            auto kstep = [&](auto bc) {
                constexpr int B = decltype(bc)::value;
                uint32_t kf0[2][2], kf1[2][2];
                k_block_frags<KVT, B>(k0, tq, kf0);
                k_block_frags<KVT, B>(k1, tq, kf1);
#pragma unroll
                for (int f = 0; f < MF; ++f)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint4 aq = qfrag[(f * (D / 16) + 2 * B + hh) * 32];
                        const uint32_t a[4] = {aq.x, aq.y, aq.z, aq.w};
                        mma16816(sacc[f][0], a, kf0[hh][0], kf0[hh][1]);
                        mma16816(sacc[f][1], a, kf1[hh][0], kf1[hh][1]);
                    }
            };
            kstep(std::integral_constant<int, 0>{});
            if constexpr (NB > 1) kstep(std::integral_constant<int, (NB > 1 ? 1 : 0)>{});
            if constexpr (NB > 2) {
                kstep(std::integral_constant<int, (NB > 2 ? 2 : 0)>{});
                kstep(std::integral_constant<int, (NB > 2 ? 3 : 0)>{});
            }
            static_assert(NB == 1 || NB == 2 || NB == 4, "slices of 1, 2 or 4 blocks");
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);                // V is in registers, K consumed: stage free

            if constexpr (NS > 1) {
                // ---- sum the NS slice partials of this cell group, in slice order
                float4 *xb = xbuf + (((i & 1) * NCG + cg) * NS) * MF * 2 * 32;
#pragma unroll
                for (int f = 0; f < MF; ++f) {
                    xb[((s * MF + f) * 2 + 0) * 32 + lane] = make_float4(sacc[f][0][0], sacc[f][0][1], sacc[f][0][2], sacc[f][0][3]);
                    xb[((s * MF + f) * 2 + 1) * 32 + lane] = make_float4(sacc[f][1][0], sacc[f][1][1], sacc[f][1][2], sacc[f][1][3]);
                }
                asm volatile("bar.sync %0, %1;" ::"r"(3 + cg), "n"(NS * 32) : "memory");
#pragma unroll
                for (int f = 0; f < MF; ++f)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        float4 acc = xb[((0 * MF + f) * 2 + nt) * 32 + lane];
#pragma unroll
                        for (int s2 = 1; s2 < NS; ++s2) {
                            const float4 v = xb[((s2 * MF + f) * 2 + nt) * 32 + lane];
                            acc.x += v.x, acc.y += v.y, acc.z += v.z, acc.w += v.w;
                        }
                        sacc[f][nt][0] = acc.x, sacc[f][nt][1] = acc.y, sacc[f][nt][2] = acc.z, sacc[f][nt][3] = acc.w;
                    }
            }

            // Mask only where a key can fall past the chunk end or a row's causal
            // limit (the last n_q - 1 keys of the sequence); the test is warp-uniform.
            // Fold-padding rows (r >= M, zero Q) are then unmasked in most tiles: their
            // partials stay finite and are never read.
            const int key0 = c_begin + kw0;
            if (key0 + 16 > c_end || key0 + 15 > sq.n_kv - sq.n_q) {
#pragma unroll
                for (int f = 0; f < MF; ++f)
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int lim = row_t[f][hr] < 0 ? -1 : sq.n_kv - sq.n_q + row_t[f][hr];
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int key = key0 + nt * 8 + 2 * tq + e;
                                if (key >= c_end || key > lim) sacc[f][nt][2 * hr + e] = -INFINITY;
                            }
                    }
            }
            // Online softmax with a lazy rescale: the running max m_r moves (and O, l
            // are rescaled) only when a tile raises it by more than kLazy (log2 units);
            // otherwise p = exp2(s - m_r) <= 2^kLazy, which f16 and the f32 sums hold.
            // (m_r, l_r, O) stay one consistent partial either way.
            constexpr float kLazy = 8.f;
            uint32_t pa[MF][4];
#pragma unroll
            for (int f = 0; f < MF; ++f)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    float mx = fmaxf(fmaxf(sacc[f][0][2 * hr], sacc[f][0][2 * hr + 1]),
                                     fmaxf(sacc[f][1][2 * hr], sacc[f][1][2 * hr + 1]));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    if (mx > m_r[f][hr] + kLazy) {   // also the first finite max (m_r = -inf)
                        const float alpha = (m_r[f][hr] == -INFINITY) ? 0.f : fast_exp2(m_r[f][hr] - mx);
                        m_r[f][hr] = mx;
                        l_r[f][hr] *= alpha;
#pragma unroll
                        for (int i2 = 0; i2 < ND; ++i2) {
                            o[f][i2][2 * hr] *= alpha;
                            o[f][i2][2 * hr + 1] *= alpha;
                        }
                    }
                    const float msafe = (m_r[f][hr] == -INFINITY) ? 0.f : m_r[f][hr];
                    const float p00 = fast_exp2(sacc[f][0][2 * hr] - msafe), p01 = fast_exp2(sacc[f][0][2 * hr + 1] - msafe);
                    const float p10 = fast_exp2(sacc[f][1][2 * hr] - msafe), p11 = fast_exp2(sacc[f][1][2 * hr + 1] - msafe);
                    l_r[f][hr] += (p00 + p01) + (p10 + p11);
                    pa[f][hr] = h2_bits(__floats2half2_rn(p00, p01));
                    pa[f][2 + hr] = h2_bits(__floats2half2_rn(p10, p11));
                }

            // ---- O += P V: b0 from cells (2t, 2t+1), b1 from (2t+8, 2t+9), slice dims KS/8*g + nd
            const __half2 s01 = bits_h2(__byte_perm(vc[0].sw, vc[1].sw, spair));
            const __half2 s89 = bits_h2(__byte_perm(vc[2].sw, vc[3].sw, spair));
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                uint32_t x01 = vc[0].d[w], y01 = vc[1].d[w], x89 = vc[2].d[w], y89 = vc[3].d[w];
                if constexpr (KVT == ARC_KV_Q4_0) {
                    x01 = (x01 >> vsh) & 0x0F0F0F0Fu, y01 = (y01 >> vsh) & 0x0F0F0F0Fu;
                    x89 = (x89 >> vsh) & 0x0F0F0F0Fu, y89 = (y89 >> vsh) & 0x0F0F0F0Fu;
                }
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t sel = half ? 0x7362u : 0x5140u;   // bytes 2,3 or 0,1 of both cells, interleaved
                    __half2 a0, a1, c0, c1;
                    if constexpr (KVT == ARC_KV_Q8_0) {
                        s8x4_to_h2x2(__byte_perm(x01, y01, sel), a0, a1);
                        s8x4_to_h2x2(__byte_perm(x89, y89, sel), c0, c1);
                    } else {
                        u4x4_to_h2x2(__byte_perm(x01, y01, sel), a0, a1);
                        u4x4_to_h2x2(__byte_perm(x89, y89, sel), c0, c1);
                    }
                    const int nd = 4 * w + 2 * half;
                    const uint32_t b00 = h2_bits(__hmul2(a0, s01)), b01 = h2_bits(__hmul2(c0, s89));
                    const uint32_t b10 = h2_bits(__hmul2(a1, s01)), b11 = h2_bits(__hmul2(c1, s89));
#pragma unroll
                    for (int f = 0; f < MF; ++f) {
                        mma16816(o[f][nd], pa[f], b00, b01);
                        mma16816(o[f][nd + 1], pa[f], b10, b11);
                    }
                }
            }
        }
        if (!ok && lane == 0) report(p.status, ST_TIMEOUT_LOAD);
#pragma unroll
        for (int f = 0; f < MF; ++f)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                l_r[f][hr] += __shfl_xor_sync(0xffffffffu, l_r[f][hr], 1);
                l_r[f][hr] += __shfl_xor_sync(0xffffffffu, l_r[f][hr], 2);
            }
    }

    // ---- merge the 4 consumer warps (the raw ring is idle now).  The producer warp arrives
    // whole (its lane 0 ran the load loop alone), so the merge's first barrier holds until
    // every consumer warp is past its last read of the ring.
    __syncwarp();
    write_ws_partial<KVT, D, MF>(o, m_r, l_r, cg, s, warp < 4, smem, p, part_index(p, s_idx, kvh, rg, sp));
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Merge the chunk partials of one (sequence, kv head, fold row) by their
// log-sum-exp weights, normalise, write O and LSE.  blockIdx.y is the fold row
// (row group * rows + row within the group).
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const __grid_constant__ DecodeParams p)
{
    __shared__ float s_w[256];     // per-split weight exp2(m_sp - m)
    __shared__ float s_m[256], s_l[256];
    __shared__ float s_red[2];
    const int s = blockIdx.x / p.Hkv, kvh = blockIdx.x % p.Hkv, r = blockIdx.y;
    const arc_seq sq = p.seqs[s];
    const int G = p.H / p.Hkv;
    if (r >= G * sq.n_q) return;
    const int h = kvh * G + r / sq.n_q, tok = sq.q_begin + r % sq.n_q;
    const int d = threadIdx.x;
    const int R = p.rows, rl = r % R;
    const int64_t part0 = part_index(p, s, kvh, r / R, 0);
    asm volatile("griddepcontrol.wait;" ::: "memory");  // partials of the split kernel are complete
    // This thread's column of the first KV32 splits goes out at once, with every
    // split's (max, sum); warp 0 reduces the latter while those loads fly.
    constexpr int KV32 = 32;
    const int nsp = p.splits;
    float v[KV32];
#pragma unroll
    for (int sp = 0; sp < KV32; ++sp)
        v[sp] = sp < nsp ? __ldcg(p.ws_o + ((part0 + sp) * R + rl) * D + d) : 0.f;
    for (int sp = d; sp < nsp; sp += D) {
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.ws_ml + ((part0 + sp) * R + rl) * 2));
        s_m[sp] = ml.x;
        s_l[sp] = ml.y;
    }
    __syncthreads();
    if (d < 32) {
        float mm = -INFINITY;
        for (int sp = d; sp < nsp; sp += 32) mm = fmaxf(mm, s_m[sp]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
        const float ms = (mm == -INFINITY) ? 0.f : mm;
        float ll = 0.f;
        for (int sp = d; sp < nsp; sp += 32) {
            const float f = (s_m[sp] == -INFINITY) ? 0.f : exp2f(s_m[sp] - ms);
            s_w[sp] = f;
            ll += f * s_l[sp];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ll += __shfl_xor_sync(0xffffffffu, ll, o);
        if (d == 0) {
            s_red[0] = mm;
            s_red[1] = ll;
        }
    }
    __syncthreads();
    const float mm = s_red[0], ll = s_red[1];
    float acc = 0.f;
#pragma unroll
    for (int sp = 0; sp < KV32; ++sp) acc += s_w[sp < nsp ? sp : 0] * v[sp];   // v is 0 past nsp
#pragma unroll 4
    for (int sp = KV32; sp < nsp; ++sp) acc += s_w[sp] * __ldcg(p.ws_o + ((part0 + sp) * R + rl) * D + d);
    p.o[((int64_t)tok * p.H + h) * D + d] = ll > 0.f ? acc / ll : 0.f;
    if (d == 0) p.lse[(int64_t)tok * p.H + h] = ll > 0.f ? (mm + log2f(ll)) * LN2 : -INFINITY;
}

// The merge launches as a programmatic dependent: its launch overlaps the split
// kernel's tail and it waits (griddepcontrol.wait) for the partials.
template <int D>
cudaError_t launch_combine(const DecodeParams &p, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_seq * p.Hkv, p.rows * p.row_groups);
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

template <int KVT, int D, int MF>
cudaError_t launch_ws(const DecodeParams &p, cudaStream_t s)
{
    const int grid = p.n_seq * p.Hkv * p.row_groups * p.splits;
    if (grid == 0) return cudaSuccess;
    auto k1 = decode_ws_kernel<KVT, D, MF>;
    const int bytes = WsLayout<KVT, D, MF>::BYTES;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess) return e;
    k1<<<grid, WS_WARPS * 32, bytes, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_combine<D>(p, s);
}

template <int KVT, int D>
cudaError_t launch_split(const DecodeParams &p, cudaStream_t s)
{
    const int grid = p.n_seq * p.Hkv * p.splits;
    if (grid == 0) return cudaSuccess;
    auto k1 = decode_split_kernel<KVT, D, false>;
    const int bytes = DecLayout<KVT, D, false>::BYTES;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess) return e;
    k1<<<grid, WARPS * 32, bytes, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_combine<D>(p, s);
}

// Dispatch over the instantiated (cache type, head dim, fragments) of the TMA kernel.
template <typename F>
auto ws_dispatch(int kv_type, int D, int mf, F &&f)
{
#define ARC_WS(T, DD, M) \
    if (kv_type == T && D == DD && mf == M) return f(std::integral_constant<int, T>{}, std::integral_constant<int, DD>{}, std::integral_constant<int, M>{});
    ARC_WS(ARC_KV_Q8_0, 64, 1) ARC_WS(ARC_KV_Q8_0, 64, 2) ARC_WS(ARC_KV_Q8_0, 128, 1) ARC_WS(ARC_KV_Q8_0, 128, 2)
    ARC_WS(ARC_KV_Q8_0, 256, 1) ARC_WS(ARC_KV_Q8_0, 256, 2) ARC_WS(ARC_KV_Q8_0, 512, 1)
    ARC_WS(ARC_KV_Q4_0, 64, 1) ARC_WS(ARC_KV_Q4_0, 64, 2) ARC_WS(ARC_KV_Q4_0, 128, 1) ARC_WS(ARC_KV_Q4_0, 128, 2)
    ARC_WS(ARC_KV_Q4_0, 256, 1) ARC_WS(ARC_KV_Q4_0, 256, 2) ARC_WS(ARC_KV_Q4_0, 512, 1)
#undef ARC_WS
    return f(std::integral_constant<int, 0>{}, std::integral_constant<int, 0>{}, std::integral_constant<int, 0>{});
}

}  // namespace

bool decode_ws_supported(int kv_type, int D, int mf)
{
    return ws_dispatch(kv_type, D, mf, [](auto t, auto d, auto m) { return decltype(d)::value != 0; });
}

int decode_smem_bytes(int kv_type, int D, int mf, bool tma)
{
    if (tma)
        return ws_dispatch(kv_type, D, mf, [](auto t, auto d, auto m) {
            if constexpr (decltype(d)::value == 0) return 0;
            else return WsLayout<decltype(t)::value, decltype(d)::value, decltype(m)::value>::BYTES;
        });
    if (kv_type == ARC_KV_Q8_0)
        return D == 64 ? DecLayout<ARC_KV_Q8_0, 64, false>::BYTES : DecLayout<ARC_KV_Q8_0, 128, false>::BYTES;
    return D == 64 ? DecLayout<ARC_KV_Q4_0, 64, false>::BYTES : DecLayout<ARC_KV_Q4_0, 128, false>::BYTES;
}

// CTAs of the split kernel that fit on one SM at once (registers, threads and
// shared memory together), from the occupancy API; 0 if it cannot be asked (no device).
int decode_blocks_per_sm(int kv_type, int D, int mf, bool tma)
{
    int n = 0;
    const int smem = decode_smem_bytes(kv_type, D, mf, tma);
    auto ask = [&](auto kern, int threads) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
    };
    const bool q8 = kv_type == ARC_KV_Q8_0;
    if (tma) {
        ws_dispatch(kv_type, D, mf, [&](auto t, auto d, auto m) {
            if constexpr (decltype(d)::value != 0)
                ask(decode_ws_kernel<decltype(t)::value, decltype(d)::value, decltype(m)::value>, WS_WARPS * 32);
            return 0;
        });
    } else {
        if (q8)
            D == 64 ? ask(decode_split_kernel<ARC_KV_Q8_0, 64, false>, WARPS * 32)
                    : ask(decode_split_kernel<ARC_KV_Q8_0, 128, false>, WARPS * 32);
        else
            D == 64 ? ask(decode_split_kernel<ARC_KV_Q4_0, 64, false>, WARPS * 32)
                    : ask(decode_split_kernel<ARC_KV_Q4_0, 128, false>, WARPS * 32);
    }
    return n;
}

// TMA box of the split kernel: {width in bytes, cells}; the width covers one head-dim
// slice of a head row from the 16-byte boundary at or below it.
void decode_box(int kv_type, int D, int mf, int *width, int *cells)
{
    *width = *cells = 0;
    ws_dispatch(kv_type, D, mf, [&](auto t, auto d, auto m) {
        if constexpr (decltype(d)::value != 0) {
            *width = WsLayout<decltype(t)::value, decltype(d)::value, decltype(m)::value>::RS;
            *cells = WsShape<decltype(d)::value, decltype(m)::value>::DT;
        }
        return 0;
    });
}

cudaError_t launch_decode(const DecodeParams &p, cudaStream_t s)
{
    if (p.splits > 256 || p.rows != 16 * p.mf) return cudaErrorInvalidValue;
    if (p.tma)
        return ws_dispatch(p.kv_type, p.D, p.mf, [&](auto t, auto d, auto m) -> cudaError_t {
            if constexpr (decltype(d)::value == 0) return cudaErrorInvalidValue;
            else return launch_ws<decltype(t)::value, decltype(d)::value, decltype(m)::value>(p, s);
        });
    if (p.mf != 1 || p.row_groups != 1) return cudaErrorInvalidValue;
    if (p.kv_type == ARC_KV_Q8_0) {
        if (p.D == 64) return launch_split<ARC_KV_Q8_0, 64>(p, s);
        if (p.D == 128) return launch_split<ARC_KV_Q8_0, 128>(p, s);
    } else {
        if (p.D == 64) return launch_split<ARC_KV_Q4_0, 64>(p, s);
        if (p.D == 128) return launch_split<ARC_KV_Q4_0, 128>(p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace arc
