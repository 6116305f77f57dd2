// attn_bwd.cu -- backward of the fused attention forward (dense / GQA fold, sinks)
// on tcgen05 tensor cores: dQ, dK, dV and the sink gradient from Q, K, V, O, dO
// and the forward's LSE.
//
// The gradients are the derivative of the forward definition.  With
// S = scale * Q K^T (masked entries -inf), P = exp(S - LSE) (the LSE includes the
// sink, so P is the forward's softmax), D_i = sum_d dO_id O_id and an optional
// upstream dLSE:
//     dV = P^T dO        dP = dO V^T        dS = P * (dP - (D_i - dLSE_i))
//     dQ = scale dS K    dK = scale dS^T Q  d sink_h = -sum_i exp(sink_h - LSE_i) (D_i - dLSE_i)
// "TransformerEngine: FA4 in context-parallel attention" (flowchart) runs FA4's
// raw backward per chunk in this form: P and D are rebuilt from the saved O and
// LSE.  GQA sums dK, dV over the g query heads of a kv head; here that sum is a
// loop over the kv group's g*Tq fold rows (the fold of "ArcFlash ... rung 0"),
// inside one accumulator, with no atomics.
//
// Kernels (every wait bounded; a wait that runs out reports through p.status):
//   bwd_prep_kernel   delta_i = D_i - dLSE_i, a warp per few rows (HBM-bound)
//   bwd_dsink_kernel  one CTA per head: the sink gradient, a fixed-order sum
//   bwd_dkdv_kernel   one CTA per (128-key tile, batch, kv head[, row split]), key tiles
//                     outermost so the causally heaviest CTAs start first:
//                       S^T  = K Q^T       M=128 keys, N=64 fold rows (a half tile)
//                       dP^T = V dO^T
//                       P^T, dS^T from S^T, dP^T, LSE, delta (two groups of softmax
//                       warps, a 32-row chunk each), written back over the chunk's
//                       own S^T / dP^T columns as bf16 (TMEM A operands)
//                       dV  += P^T dO      dK += dS^T Q   (dO, Q read MN-major)
//                     TMEM: dV [0, DV), dK [DV, DV+D), then S^T / dP^T of each half;
//                     the two halves of a 128-row fold tile alternate, so one half's
//                     softmax overlaps the other half's products (one half of 64
//                     rows per tile at d_qk 192, where TMEM has no room for two)
//   bwd_dq_kernel     one CTA per (batch, kv head, 128-row fold tile), the tiles in
//                     order of decreasing causal work (a host-sorted table):
//                       S = Q K^T, dP = dO V^T, dS (softmax warps, over S),
//                       dQ += dS K         (K read MN-major)
//                     TMEM: dQ [0, D), S / dP of two 64-key halves at 256 and 384,
//                     alternating like the dK / dV halves
//   bwd_reduce_kernel the fp32 partials of row-split dK/dV CTAs, summed in order
// S and dP are computed in both main kernels (5 + 2 products per tile pair for
// 5 algorithmic): the price of needing no atomics and no dS round trip
// through memory.
#include <limits.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace arc {
namespace {

constexpr int BK = 128;                 // keys per tile (dK/dV: the CTA's keys; dQ: the streamed tile)
constexpr int BQ = 128;                 // fold rows per dQ tile
constexpr int KCH = 128 * 128;          // bytes of a [128 rows x 64 bf16] swizzled chunk
constexpr int BW_THREADS = 256;         // dQ: producer, MMA issuer, 2 idle, 4 softmax / epilogue warps
// dK/dV: producer, MMA issuer, 2 idle, then two groups of 4 softmax / epilogue warps (two
// warps per lane quadrant), each group taking every other 32-row chunk of a half, so the
// TMEM load -> exp2 -> TMEM store chains of two chunks overlap
constexpr int DKDV_GROUPS = 2;
constexpr int DKDV_THREADS = 128 + DKDV_GROUPS * 128;
constexpr int BW_SMEM_LIMIT = 232448;
constexpr float BW_LOG2E = 1.4426950408889634f;

struct BwdBars {
    uint64_t fixed_full;        // the CTA's resident operands (dK/dV: K, V; dQ: Q, dO)
    uint64_t full[2], empty[2]; // two-stage ring of the streamed operand tiles
    uint64_t s_full[2];         // S and dP of a half are in TMEM
    uint64_t p_full[2];         // the softmax warps wrote P / dS of a half (128 arrivals)
    uint64_t done;              // every MMA of the CTA finished
    uint64_t cols;              // dK/dV: a fold tile's row quantities are in shared memory (128 arrivals)
    uint32_t tmem_base;
};

// Where a bounded wait of the backward ran out (OR-ed into the status word beside
// the role's ST_TIMEOUT_* code).
enum : uint32_t {
    BW_AT_FIXED = 1u << 8,
    BW_AT_RING_EMPTY = 1u << 9,
    BW_AT_RING_FULL = 1u << 10,
    BW_AT_S_FULL = 1u << 11,
    BW_AT_P_FULL = 1u << 12,
    BW_AT_COLS = 1u << 13,
    BW_AT_DONE = 1u << 14,
    BW_IN_DQ = 1u << 15,        // the wait was in the dQ kernel (else dK / dV)
};

__device__ __forceinline__ bool bw_all(bool ok) { return __all_sync(0xffffffffu, ok); }

// Does fold tile qt (rows qt*BR .. of the kv group) see any key at or after k0?
__device__ __forceinline__ bool q_tile_live(const BwdParams &p, int qt, int BR, int k0)
{
    if (!p.causal) return true;
    const int rows = p.G * p.Tq;
    const int r0 = qt * BR, r_last = min(r0 + BR, rows) - 1;
    const int t_max = (r0 / p.Tq != r_last / p.Tq) ? p.Tq - 1 : r_last % p.Tq;
    return t_max + p.Tk - p.Tq >= k0;
}

// The per-row quantities of fold row r of kv head kvh: LSE in log2 units (+inf for a
// row that sees nothing, so its P is 0), delta, and the last key it may see.
struct RowInfo {
    float lse2, delta;
    int lim;
};

__device__ __forceinline__ RowInfo row_info(const BwdParams &p, int b, int kvh, int r)
{
    RowInfo ri{INFINITY, 0.f, -1};
    if (r >= p.G * p.Tq) return ri;
    const int h = kvh * p.G + r / p.Tq, t = r % p.Tq;
    const int64_t i = ((int64_t)b * p.H + h) * p.Tq + t;
    const float l = p.lse[i];
    ri.lse2 = (l == -INFINITY) ? INFINITY : l * BW_LOG2E;
    ri.delta = p.delta[i];
    ri.lim = p.causal ? min(p.Tk - 1, t + p.Tk - p.Tq) : p.Tk - 1;
    return ri;
}


static_assert(sizeof(BwdParams) <= 4096, "backward parameters fit the classic kernel-parameter space");

// dK / dV.  A fold tile of BR rows is processed as NH halves of HR = BR/NH rows, each
// with its own S^T / dP^T buffers in TMEM: while the softmax warps rebuild P and dS of
// one half, the tensor core runs the other half's products.
template <int D, int DV, int BR, int NH>
struct DkdvLayout {
    static constexpr int KC = D / 64, VC = DV / 64;
    static constexpr int HR = BR / NH;                        // fold rows per half
    static constexpr int QCH = BR * 128;                      // one 64-column chunk of a fold tile
    static constexpr int STAGE = (KC + VC) * QCH;             // Q and dO of one fold tile
    static constexpr int FIXED = (KC + VC) * KCH;             // K and V of the CTA's key tile
    // + per fold tile (two buffers): (LSE, delta) pairs, last visible keys, per-warp minima
    static constexpr int BYTES = 1024 + FIXED + 2 * STAGE + 2 * 128 * 12 + 2 * 4 * 4 + (int)sizeof(BwdBars);
    static constexpr int DV_COL = 0, DK_COL = DV;
    __host__ __device__ static constexpr int s_col(int h) { return DV + D + h * 2 * HR; }
    __host__ __device__ static constexpr int dp_col(int h) { return DV + D + h * 2 * HR + HR; }
    static_assert(HR % 64 == 0 && BR % HR == 0, "halves of whole 64-row K groups");
    static_assert(DV + D + NH * 2 * HR <= 512, "TMEM: dV, dK and NH pairs of S^T / dP^T side by side");
    static_assert(BYTES <= BW_SMEM_LIMIT, "shared memory");
};

template <int D, int DV, int BR, int NH>
__global__ void __launch_bounds__(DKDV_THREADS, 1) bwd_dkdv_kernel(const __grid_constant__ BwdParams p)
{
    using L = DkdvLayout<D, DV, BR, NH>;
    constexpr int KC = L::KC, VC = L::VC, HR = L::HR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem<1024>(smem_raw);
    uint8_t *sK = smem, *sV = sK + KC * KCH;
    uint8_t *sRing = sK + L::FIXED;                             // [2][Q chunks, dO chunks]
    float2 *col_ld = reinterpret_cast<float2 *>(sRing + 2 * L::STAGE);   // [2][128] (LSE in log2 units, delta)
    int *col_lim = reinterpret_cast<int *>(col_ld + 2 * 128);             // [2][128] last key a row may see
    int *col_wmin = col_lim + 2 * 128;                                    // [2][4] min of those per 32 rows
    BwdBars *bars = reinterpret_cast<BwdBars *>(col_wmin + 2 * 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // key-tile-major: under a causal mask the first key tiles see the most fold rows, so
    // the heaviest CTAs of every (batch, kv head) go out first and the light ones fill in
    const int rs = blockIdx.x % p.rsplit;
    const int kvh = (blockIdx.x / p.rsplit) % p.Hkv;
    const int b = (blockIdx.x / (p.rsplit * p.Hkv)) % p.B;
    const int kt = blockIdx.x / (p.rsplit * p.Hkv * p.B);
    const int k0 = kt * BK;
    const int n_qt = (p.G * p.Tq + BR - 1) / BR;
    const int qt_begin = rs * p.tiles_per_split, qt_end = min(n_qt, qt_begin + p.tiles_per_split);
    const int row_base = kvh * p.G * p.Tq;                      // fold row 0 in the [H*Tq] view
    // the next fold tile at or after qt that sees one of this CTA's keys (qt_end if none)
    auto next_live = [&](int qt) {
        while (qt < qt_end && !q_tile_live(p, qt, BR, k0)) ++qt;
        return qt;
    };

    if (threadIdx.x == 0) {
        mbar_init(&bars->fixed_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], 1);
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], DKDV_GROUPS * 128);
        }
        mbar_init(&bars->done, 1);
        mbar_init(&bars->cols, DKDV_GROUPS * 128);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // =============================== TMA producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars->fixed_full, L::FIXED);
            for (int c = 0; c < KC; ++c) {
                if (!p.mla || c < p.kc_first)
                    tma_load_4d(sK + c * KCH, &p.tm_k, &bars->fixed_full, c * 64, k0, kvh, b);
                else   // MLA: the rope columns, one tensor shared by every head
                    tma_load_3d(sK + c * KCH, &p.tm_k2, &bars->fixed_full, (c - p.kc_first) * 64, k0, b);
            }
            for (int c = 0; c < VC; ++c) tma_load_4d(sV + c * KCH, &p.tm_v, &bars->fixed_full, c * 64, k0, kvh, b);
            int it = 0;
            bool ok = true;
            for (int qt = next_live(qt_begin); qt < qt_end && ok; qt = next_live(qt + 1)) {
                const int st = it & 1;
                if (it >= 2) ok = mbar_wait(&bars->empty[st], (uint32_t)(((it >> 1) - 1) & 1));
                if (!ok) {
                    report(p.status, BW_AT_RING_EMPTY);
                    break;
                }
                uint8_t *dst = sRing + st * L::STAGE;
                mbar_arrive_expect_tx(&bars->full[st], L::STAGE);
                for (int c = 0; c < KC; ++c) {
                    if (!p.mla || c < p.kc_first)
                        tma_load_3d(dst + c * L::QCH, &p.tm_qr, &bars->full[st], c * 64, row_base + qt * BR, b);
                    else
                        tma_load_3d(dst + c * L::QCH, &p.tm_qr2, &bars->full[st], (c - p.kc_first) * 64,
                                    row_base + qt * BR, b);
                }
                for (int c = 0; c < VC; ++c)
                    tma_load_3d(dst + (KC + c) * L::QCH, &p.tm_dor, &bars->full[st], c * 64, row_base + qt * BR, b);
                ++it;
            }
            if (!ok) report(p.status, ST_TIMEOUT_LOAD);
            // every copy issued has landed before the CTA may exit
            for (int i = (it > 2 ? it - 2 : 0); i < it; ++i) mbar_wait(&bars->full[i & 1], (uint32_t)((i >> 1) & 1));
            mbar_wait(&bars->fixed_full, 0);
        }
    } else if (warp == 1) {
        // =============================== MMA issuer
        // Per fold tile and half h: S^T_h = K Q_h^T and dP^T_h = V dO_h^T (SS), then, once the
        // softmax warps have posted P^T_h / dS^T_h, dV += P^T_h dO_h and dK += dS^T_h Q_h (TS).
        // The next tile's S^T_h / dP^T_h go out right after this tile's dV / dK of the same
        // half (the tensor core runs them in issue order, so they overwrite the half's
        // columns only after those have been read), before waiting on the other half.
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16(128, HR, false, false);
            const uint32_t idesc_dv = idesc_bf16(128, DV, false, true);
            const uint32_t idesc_dk = idesc_bf16(128, D, false, true);
            const uint64_t kd0 = sdesc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t vd0 = sdesc_sw128(smem_u32(sV), 16, 1024);
            constexpr uint32_t kHalf = HR * 128 >> 4;              // descriptor units of HR rows
            bool ok = mbar_wait(&bars->fixed_full, 0);
            if (!ok) report(p.status, BW_AT_FIXED);
            tc_fence_after();
            auto issue_s = [&](int st, int h) {
                uint8_t *sq = sRing + st * L::STAGE, *sdo = sq + KC * L::QCH;
                const uint64_t qd = sdesc_sw128(smem_u32(sq), 16, 1024) + h * kHalf;
                const uint64_t dod = sdesc_sw128(smem_u32(sdo), 16, 1024) + h * kHalf;
#pragma unroll
                for (int c = 0; c < KC; ++c)
                    umma_ss_k64(tmem + L::s_col(h), kd0 + (uint64_t)(c * (KCH >> 4)),
                                qd + (uint64_t)(c * (L::QCH >> 4)), idesc_s, c > 0);
#pragma unroll
                for (int c = 0; c < VC; ++c)
                    umma_ss_k64(tmem + L::dp_col(h), vd0 + (uint64_t)(c * (KCH >> 4)),
                                dod + (uint64_t)(c * (L::QCH >> 4)), idesc_s, c > 0);
                umma_commit(&bars->s_full[h]);
            };
            int it = 0;
            int qt = next_live(qt_begin);
            if (qt < qt_end) {
                if (!(ok = ok && mbar_wait(&bars->full[0], 0))) report(p.status, BW_AT_RING_FULL);
                tc_fence_after();
                if (ok)
                    for (int h = 0; h < NH; ++h) issue_s(0, h);
            }
            for (; qt < qt_end && ok; ++it) {
                const int st = it & 1;
                const int qn = next_live(qt + 1);
                uint8_t *sq = sRing + st * L::STAGE, *sdo = sq + KC * L::QCH;
                const uint64_t dob = sdesc_sw128(smem_u32(sdo), L::QCH, 1024);
                const uint64_t qb = sdesc_sw128(smem_u32(sq), L::QCH, 1024);
#pragma unroll 1
                for (int h = 0; h < NH && ok; ++h) {
                    if (!(ok = mbar_wait(&bars->p_full[h], (uint32_t)(it & 1)))) {
                        report(p.status, BW_AT_P_FULL);
                        break;
                    }
                    tc_fence_after();
                    // dV += P^T_h dO_h, dK += dS^T_h Q_h: B read MN-major from the half's rows
                    // (16 fold rows = 2048 B per K step).  The bf16 P^T / dS^T of 32-row chunk
                    // c sit in the first 16 of that chunk's 32 columns.
                    const uint32_t acc = (it > 0 || h > 0) ? 1u : 0u;
#pragma unroll
                    for (int c2 = 0; c2 < HR / 32; ++c2)
                        umma_ts_k32(tmem + L::DV_COL, tmem + L::s_col(h) + c2 * 32,
                                    dob + (uint64_t)(h * kHalf + c2 * 256), 128, idesc_dv, acc | c2);
#pragma unroll
                    for (int c2 = 0; c2 < HR / 32; ++c2)
                        umma_ts_k32(tmem + L::DK_COL, tmem + L::dp_col(h) + c2 * 32,
                                    qb + (uint64_t)(h * kHalf + c2 * 256), 128, idesc_dk, acc | c2);
                    if (h == NH - 1) umma_commit(&bars->empty[st]);   // the stage is free once these have read it
                    if (qn < qt_end) {
                        if (h == 0) {
                            if (!(ok = mbar_wait(&bars->full[(it + 1) & 1], (uint32_t)(((it + 1) >> 1) & 1)))) {
                                report(p.status, BW_AT_RING_FULL);
                                break;
                            }
                            tc_fence_after();
                        }
                        issue_s((it + 1) & 1, h);
                    }
                }
                qt = qn;
            }
            if (!ok) report(p.status, ST_TIMEOUT_MMA);
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0);
        }
    } else if (warp >= 4) {
        // =============================== P^T, dS^T (one thread per key and chunk group) and the epilogue
        const int tid = (threadIdx.x - 128) & 127;              // key lane 0..127 (the warp's TMEM quadrant)
        const int grp = (threadIdx.x - 128) >> 7;               // chunk group
        const int kj = k0 + tid;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const float sl2 = p.scale_log2;
        int it = 0;
        bool ok = true;
        for (int qt = next_live(qt_begin); qt < qt_end; qt = next_live(qt + 1)) {
            const int cb = (it & 1) * 128;
            int lim_min = INT_MAX;    // a row past the group has P = 0 (LSE +inf) and bounds nothing
            if (grp == 0 && tid < BR) {
                const RowInfo ri = row_info(p, b, kvh, qt * BR + tid);
                col_ld[cb + tid] = make_float2(ri.lse2, ri.delta);
                col_lim[cb + tid] = ri.lim;
                if (qt * BR + tid < p.G * p.Tq) lim_min = ri.lim;
            }
            lim_min = __reduce_min_sync(0xffffffffu, lim_min);
            if (grp == 0 && lane == 0 && tid < BR) col_wmin[(it & 1) * 4 + (tid >> 5)] = lim_min;
            // every softmax thread has written its column (a bounded wait, unlike a named
            // barrier, so a thread that stopped early cannot hold the others forever)
            mbar_arrive(&bars->cols);
            ok = bw_all(mbar_wait(&bars->cols, (uint32_t)(it & 1)));
            if (!ok) {
                report(p.status, BW_AT_COLS);
                break;
            }
            // Every row of the tile sees every valid key of the CTA: no causal test per
            // element.  (A key past Tk then gets a nonzero P, but it only feeds its own
            // dK / dV rows, which are never stored.)
            int tile_min = INT_MAX;
#pragma unroll
            for (int w = 0; w < BR / 32; ++w) tile_min = min(tile_min, col_wmin[(it & 1) * 4 + w]);
            const bool whole = tile_min >= min(k0 + BK - 1, p.Tk - 1);
#pragma unroll 1
            for (int h = 0; h < NH && ok; ++h) {
                ok = bw_all(mbar_wait(&bars->s_full[h], (uint32_t)(it & 1)));
                if (!ok) {
                    report(p.status, BW_AT_S_FULL);
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int ch = grp; ch < HR / 32; ch += DKDV_GROUPS) {
                    uint32_t sv[32], dv[32];
                    tmem_ld32(tmem + lane_off + L::s_col(h) + 32 * ch, sv);
                    tmem_ld32(tmem + lane_off + L::dp_col(h) + 32 * ch, dv);
                    tmem_wait_ld();
                    const int c0 = cb + h * HR + 32 * ch;
                    uint32_t pk[16], dk[16];
                    if (whole) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float pp[2], dd[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float2 ld = col_ld[c0 + 2 * i + e];
                                pp[e] = fast_exp2(fmaf(__uint_as_float(sv[2 * i + e]), sl2, -ld.x));
                                dd[e] = pp[e] * (__uint_as_float(dv[2 * i + e]) - ld.y);
                            }
                            pk[i] = pack_bf16(pp[0], pp[1]);
                            dk[i] = pack_bf16(dd[0], dd[1]);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float pp[2], dd[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int c = c0 + 2 * i + e;
                                const float2 ld = col_ld[c];
                                const float pe =
                                    kj <= col_lim[c] ? fast_exp2(fmaf(__uint_as_float(sv[2 * i + e]), sl2, -ld.x)) : 0.f;
                                pp[e] = pe;
                                dd[e] = pe * (__uint_as_float(dv[2 * i + e]) - ld.y);
                            }
                            pk[i] = pack_bf16(pp[0], pp[1]);
                            dk[i] = pack_bf16(dd[0], dd[1]);
                        }
                    }
                    // bf16 pairs over the first half of the columns just read (no other
                    // chunk group reads or writes these columns)
                    tmem_st16(tmem + lane_off + L::s_col(h) + 32 * ch, pk);
                    tmem_st16(tmem + lane_off + L::dp_col(h) + 32 * ch, dk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[h]);
            }
            if (!ok) break;
            ++it;
        }
        if (ok && it > 0) ok = bw_all(mbar_wait(&bars->done, 0));
        if (!ok) report(p.status, ST_TIMEOUT_SOFTMAX);
        tc_fence_after();
        // ---- epilogue: dV and scale * dK of key kj (fp32 partials under a row split).
        // The TMEM loads are warp-collective: every lane loads, only keys < Tk store.
        const bool live = it > 0 && ok;
        const bool key_ok = kj < p.Tk;
        float *prow = p.dkv_part + ((((int64_t)rs * p.B + b) * p.Hkv + kvh) * p.Tk + kj) * (D + DV);
        __nv_bfloat16 *dkrow = p.dk + (int64_t)b * p.dks[0] + (int64_t)kvh * p.dks[1] + (int64_t)kj * p.dks[2];
        __nv_bfloat16 *dvrow = p.dv + (int64_t)b * p.dvs[0] + (int64_t)kvh * p.dvs[1] + (int64_t)kj * p.dvs[2];
        const int dr = D - p.dk_cols;                             // MLA: rope columns of dK (else 0)
        float *rrow = p.dkr_part + ((((int64_t)rs * p.B + b) * p.Hkv + kvh) * p.Tk + kj) * dr;
#pragma unroll 1
        for (int c = grp; c < (D + DV) / 32; c += DKDV_GROUPS) {
            uint32_t v[32];
            const bool is_k = c < D / 32;
            const int col = is_k ? L::DK_COL + 32 * c : L::DV_COL + 32 * (c - D / 32);
            if (live) {
                tmem_ld32(tmem + lane_off + col, v);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0u;
            }
            if (!key_ok) continue;
            if (is_k && 32 * c >= p.dk_cols) {
                // MLA rope columns: this head's share of the shared k_rope's gradient (fp32,
                // unscaled); a reduction sums the heads
                float4 *dst = reinterpret_cast<float4 *>(rrow + 32 * c - p.dk_cols);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                         __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
                continue;
            }
            if (p.rsplit > 1) {
                float4 *dst = reinterpret_cast<float4 *>(prow + 32 * c);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                         __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            } else {
                const float f = is_k ? p.scale : 1.f;
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16(__uint_as_float(v[2 * i]) * f, __uint_as_float(v[2 * i + 1]) * f);
                uint4 *dst = reinterpret_cast<uint4 *>(is_k ? dkrow + 32 * c : dvrow + 32 * (c - D / 32));
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
    }

    // Each warp arrives whole (a role branch may have left lanes behind, e.g. the MMA
    // issuer's lane 0), so the barrier below holds until every warp is done with TMEM.
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dQ.  A key tile of 128 keys is processed as two halves of 64 keys, each with its own
// S / dP buffers in TMEM, pipelined like the dK / dV kernel's halves.
template <int D, int DV>
struct DqLayout {
    static constexpr int KC = D / 64, VC = DV / 64;
    static constexpr int FIXED = (KC + VC) * KCH;             // Q and dO of the CTA's fold tile
    static constexpr int STAGE = (KC + VC) * KCH;             // K and V of one key tile
    // two ring stages where they fit beside Q and dO, else one (d 192: the next key
    // tile then loads only once the last one is consumed)
    static constexpr int NSTG = 1024 + FIXED + 2 * STAGE + (int)sizeof(BwdBars) <= BW_SMEM_LIMIT ? 2 : 1;
    static constexpr int BYTES = 1024 + FIXED + NSTG * STAGE + (int)sizeof(BwdBars);
    static constexpr int DQ_COL = 0;
    __host__ __device__ static constexpr int s_col(int h) { return 256 + h * 128; }
    __host__ __device__ static constexpr int dp_col(int h) { return 256 + h * 128 + 64; }
    static_assert(D <= 256, "TMEM: dQ, then two pairs of S / dP halves");
    static_assert(BYTES <= BW_SMEM_LIMIT, "shared memory");
};

template <int D, int DV>
__global__ void __launch_bounds__(BW_THREADS, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p)
{
    using L = DqLayout<D, DV>;
    constexpr int KC = L::KC, VC = L::VC, HK = BK / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem<1024>(smem_raw);
    uint8_t *sQ = smem, *sdO = sQ + KC * KCH;
    uint8_t *sRing = smem + L::FIXED;                           // [NSTG][K chunks, V chunks]
    BwdBars *bars = reinterpret_cast<BwdBars *>(sRing + L::NSTG * L::STAGE);
    constexpr int NS = L::NSTG;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows = p.G * p.Tq;
    const int n_rt = (rows + BQ - 1) / BQ;
    // heavier tiles (later positions see more keys) first, over all (batch, kv head) pairs
    const int nbh = p.B * p.Hkv;
    const int rank = blockIdx.x / nbh;
    const int rt = p.dq_order_n ? (int)p.dq_order[rank] : n_rt - 1 - rank;
    const int kvh = (blockIdx.x % nbh) % p.Hkv;
    const int b = (blockIdx.x % nbh) / p.Hkv;
    const int r0 = rt * BQ;
    int nt;
    {
        const int r_last = min(r0 + BQ, rows) - 1;
        const int t_max = (r0 / p.Tq != r_last / p.Tq) ? p.Tq - 1 : r_last % p.Tq;
        const int kv_last = p.causal ? min(p.Tk - 1, t_max + p.Tk - p.Tq) : p.Tk - 1;
        nt = kv_last < 0 ? 0 : kv_last / BK + 1;
    }
    const int row_base = kvh * rows;

    if (threadIdx.x == 0) {
        mbar_init(&bars->fixed_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], 1);
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 128);
        }
        mbar_init(&bars->done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // =============================== TMA producer
        if (lane == 0 && nt > 0) {
            mbar_arrive_expect_tx(&bars->fixed_full, L::FIXED);
            for (int c = 0; c < KC; ++c) {
                if (!p.mla || c < p.kc_first)
                    tma_load_3d(sQ + c * KCH, &p.tm_q, &bars->fixed_full, c * 64, row_base + r0, b);
                else
                    tma_load_3d(sQ + c * KCH, &p.tm_q2, &bars->fixed_full, (c - p.kc_first) * 64, row_base + r0, b);
            }
            for (int c = 0; c < VC; ++c) tma_load_3d(sdO + c * KCH, &p.tm_do, &bars->fixed_full, c * 64, row_base + r0, b);
            bool ok = true;
            for (int j = 0; j < nt && ok; ++j) {
                const int st = j % NS;
                if (j >= NS) ok = mbar_wait(&bars->empty[st], (uint32_t)((j / NS - 1) & 1));
                if (!ok) {
                    report(p.status, BW_IN_DQ | BW_AT_RING_EMPTY);
                    break;
                }
                uint8_t *dst = sRing + st * L::STAGE;
                mbar_arrive_expect_tx(&bars->full[st], L::STAGE);
                for (int c = 0; c < KC; ++c) {
                    if (!p.mla || c < p.kc_first)
                        tma_load_4d(dst + c * KCH, &p.tm_k, &bars->full[st], c * 64, j * BK, kvh, b);
                    else
                        tma_load_3d(dst + c * KCH, &p.tm_k2, &bars->full[st], (c - p.kc_first) * 64, j * BK, b);
                }
                for (int c = 0; c < VC; ++c)
                    tma_load_4d(dst + (KC + c) * KCH, &p.tm_v, &bars->full[st], c * 64, j * BK, kvh, b);
            }
            if (!ok) report(p.status, ST_TIMEOUT_LOAD);
            for (int i = (nt > NS ? nt - NS : 0); i < nt; ++i) mbar_wait(&bars->full[i % NS], (uint32_t)((i / NS) & 1));
            mbar_wait(&bars->fixed_full, 0);
        }
    } else if (warp == 1) {
        // =============================== MMA issuer
        if (lane == 0 && nt > 0) {
            const uint32_t idesc_s = idesc_bf16(128, HK, false, false);
            const uint32_t idesc_dq = idesc_bf16(128, D, false, true);
            const uint64_t qd0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dod0 = sdesc_sw128(smem_u32(sdO), 16, 1024);
            constexpr uint32_t kHalf = HK * 128 >> 4;              // descriptor units of 64 key rows
            bool ok = mbar_wait(&bars->fixed_full, 0);
            if (!ok) report(p.status, BW_IN_DQ | BW_AT_FIXED);
            tc_fence_after();
            // S_h = Q K_h^T and dP_h = dO V_h^T for key half h of key tile j (ring stage st)
            auto issue_s = [&](int st, int h) {
                uint8_t *sk = sRing + st * L::STAGE, *sv = sk + KC * KCH;
                const uint64_t kd = sdesc_sw128(smem_u32(sk), 16, 1024) + h * kHalf;
                const uint64_t vd = sdesc_sw128(smem_u32(sv), 16, 1024) + h * kHalf;
#pragma unroll
                for (int c = 0; c < KC; ++c)
                    umma_ss_k64(tmem + L::s_col(h), qd0 + (uint64_t)(c * (KCH >> 4)), kd + (uint64_t)(c * (KCH >> 4)),
                                idesc_s, c > 0);
#pragma unroll
                for (int c = 0; c < VC; ++c)
                    umma_ss_k64(tmem + L::dp_col(h), dod0 + (uint64_t)(c * (KCH >> 4)), vd + (uint64_t)(c * (KCH >> 4)),
                                idesc_s, c > 0);
                umma_commit(&bars->s_full[h]);
            };
            if (!(ok = ok && mbar_wait(&bars->full[0], 0))) report(p.status, BW_IN_DQ | BW_AT_RING_FULL);
            tc_fence_after();
            if (ok)
                for (int h = 0; h < 2; ++h) issue_s(0, h);
            for (int j = 0; j < nt && ok; ++j) {
                const int st = j % NS;
                uint8_t *sk = sRing + st * L::STAGE;
                const uint64_t kb = sdesc_sw128(smem_u32(sk), KCH, 1024);
#pragma unroll 1
                for (int h = 0; h < 2 && ok; ++h) {
                    if (!(ok = mbar_wait(&bars->p_full[h], (uint32_t)(j & 1)))) {
                        report(p.status, BW_IN_DQ | BW_AT_P_FULL);
                        break;
                    }
                    tc_fence_after();
                    // dQ += dS_h K_h: dS from TMEM, K read MN-major (16 keys = 2048 B per K step)
                    umma_ts_k64(tmem + L::DQ_COL, tmem + L::s_col(h), kb + (uint64_t)(h * kHalf), 128, idesc_dq,
                                (j > 0 || h > 0) ? 1u : 0u);
                    if (h == 1) umma_commit(&bars->empty[st]);
                    // the next key tile's half h, right behind this half's dQ; with one ring
                    // stage the next tile can only have landed once this tile is released,
                    // so both of its halves follow the second half
                    if (j + 1 < nt && (NS > 1 || h == 1)) {
                        if (NS > 1 ? h == 0 : true) {
                            if (!(ok = mbar_wait(&bars->full[(j + 1) % NS], (uint32_t)(((j + 1) / NS) & 1)))) {
                                report(p.status, BW_IN_DQ | BW_AT_RING_FULL);
                                break;
                            }
                            tc_fence_after();
                        }
                        if (NS > 1) {
                            issue_s((j + 1) % NS, h);
                        } else {
                            issue_s(0, 0);
                            issue_s(0, 1);
                        }
                    }
                }
            }
            if (!ok) report(p.status, ST_TIMEOUT_MMA);
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0);
        }
    } else if (warp >= 4) {
        // =============================== dS (one thread per fold row) and the epilogue
        const int tid = threadIdx.x - 128;
        const int r = r0 + tid;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const RowInfo ri = row_info(p, b, kvh, r);
        const float sl2 = p.scale_log2;
        bool ok = true;
        for (int j = 0; j < nt && ok; ++j) {
#pragma unroll 1
            for (int h = 0; h < 2 && ok; ++h) {
                ok = bw_all(mbar_wait(&bars->s_full[h], (uint32_t)(j & 1)));
                if (!ok) {
                    report(p.status, BW_IN_DQ | BW_AT_S_FULL);
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int ch = 0; ch < HK / 32; ++ch) {
                    uint32_t sv[32], dv[32];
                    tmem_ld32(tmem + lane_off + L::s_col(h) + 32 * ch, sv);
                    tmem_ld32(tmem + lane_off + L::dp_col(h) + 32 * ch, dv);
                    tmem_wait_ld();
                    const int key0 = j * BK + h * HK + 32 * ch;
                    uint32_t dk[16];
                    // all 32 keys visible to every row of the warp (a row past the group has
                    // P = 0 from its +inf LSE): no causal test per element
                    if (__all_sync(0xffffffffu, r >= rows || key0 + 31 <= ri.lim)) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float dd[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float pe = fast_exp2(fmaf(__uint_as_float(sv[2 * i + e]), sl2, -ri.lse2));
                                dd[e] = pe * (__uint_as_float(dv[2 * i + e]) - ri.delta);
                            }
                            dk[i] = pack_bf16(dd[0], dd[1]);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float dd[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float pe = key0 + 2 * i + e <= ri.lim
                                                     ? fast_exp2(fmaf(__uint_as_float(sv[2 * i + e]), sl2, -ri.lse2))
                                                     : 0.f;
                                dd[e] = pe * (__uint_as_float(dv[2 * i + e]) - ri.delta);
                            }
                            dk[i] = pack_bf16(dd[0], dd[1]);
                        }
                    }
                    tmem_st16(tmem + lane_off + L::s_col(h) + 16 * ch, dk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[h]);
            }
        }
        if (ok && nt > 0) ok = bw_all(mbar_wait(&bars->done, 0));
        if (!ok) report(p.status, ST_TIMEOUT_SOFTMAX);
        tc_fence_after();
        // warp-collective TMEM loads by every lane; only rows of the group store
        const bool row_ok = r < rows;
        const int h = kvh * p.G + (row_ok ? r / p.Tq : 0), t = row_ok ? r % p.Tq : 0;
        __nv_bfloat16 *dqrow = p.dq + (int64_t)b * p.dqs[0] + (int64_t)h * p.dqs[1] + (int64_t)t * p.dqs[2];
        // MLA: columns from kc_first * 64 on are dq_rope's
        const int dn = p.mla ? p.kc_first * 64 : D;
        __nv_bfloat16 *dq2row = p.mla ? p.dq2 + (int64_t)b * p.dq2s[0] + (int64_t)h * p.dq2s[1] + (int64_t)t * p.dq2s[2]
                                      : nullptr;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            if (nt > 0 && ok) {
                tmem_ld32(tmem + lane_off + L::DQ_COL + 32 * c, v);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0u;
            }
            if (!row_ok) continue;
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = pack_bf16(__uint_as_float(v[2 * i]) * p.scale, __uint_as_float(v[2 * i + 1]) * p.scale);
            uint4 *dst = reinterpret_cast<uint4 *>(32 * c < dn ? dqrow + 32 * c : dq2row + (32 * c - dn));
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
    }

    // Each warp arrives whole (a role branch may have left lanes behind, e.g. the MMA
    // issuer's lane 0), so the barrier below holds until every warp is done with TMEM.
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// delta_i = sum_d dO_id O_id - dLSE_i.  A warp takes PREP_U groups of RPW = 256 / Dv rows
// (at least one row a group): each lane moves 8 elements (16 bytes) of one row per step,
// and the loads of all PREP_U groups go out before any is used, so a lane keeps
// 2 * PREP_U 16-byte loads in flight; the lanes of a row reduce with shuffles.
constexpr int PREP_U = 4;
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __grid_constant__ BwdPrepParams p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rpw = p.Dv >= 256 ? 1 : 256 / p.Dv;               // rows per group (a power of two)
    const int lpr = 32 / rpw;                                   // lanes per row
    const int64_t rows = (int64_t)p.B * p.H * p.Tq;
    const int64_t first = ((int64_t)blockIdx.x * 8 + warp) * PREP_U * rpw + lane / lpr;
    const __nv_bfloat16 *o[PREP_U], *g[PREP_U];
    bool live[PREP_U];
    float acc[PREP_U];
#pragma unroll
    for (int u = 0; u < PREP_U; ++u) {
        const int64_t row = first + (int64_t)u * rpw;
        live[u] = row < rows;
        acc[u] = 0.f;
        const int64_t rr = live[u] ? row : 0;
        const int t = (int)(rr % p.Tq), h = (int)((rr / p.Tq) % p.H), b = (int)(rr / ((int64_t)p.Tq * p.H));
        o[u] = p.o + (int64_t)b * p.os[0] + (int64_t)h * p.os[1] + (int64_t)t * p.os[2];
        g[u] = p.dout + (int64_t)b * p.dos[0] + (int64_t)h * p.dos[1] + (int64_t)t * p.dos[2];
    }
    for (int d = (lane % lpr) * 8; d < p.Dv; d += lpr * 8) {
        uint4 x[PREP_U], y[PREP_U];
#pragma unroll
        for (int u = 0; u < PREP_U; ++u) {
            x[u] = live[u] ? *reinterpret_cast<const uint4 *>(o[u] + d) : make_uint4(0u, 0u, 0u, 0u);
            y[u] = live[u] ? *reinterpret_cast<const uint4 *>(g[u] + d) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < PREP_U; ++u) {
            const uint32_t xw[4] = {x[u].x, x[u].y, x[u].z, x[u].w}, yw[4] = {y[u].x, y[u].y, y[u].z, y[u].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xw[k]));
                const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&yw[k]));
                acc[u] = fmaf(a.x, c.x, acc[u]);
                acc[u] = fmaf(a.y, c.y, acc[u]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < PREP_U; ++u) {
        for (int sh = lpr / 2; sh > 0; sh >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], sh);
        const int64_t row = first + (int64_t)u * rpw;
        if (live[u] && lane % lpr == 0) p.delta[row] = acc[u] - (p.dlse ? p.dlse[row] : 0.f);
    }
}

// d sink_h = -sum_{b,t} exp(sink_h - LSE_bht) * delta_bht, one CTA per head, a fixed
// summation order (strided per thread, then a tree), so the result is reproducible.
__global__ void __launch_bounds__(256) bwd_dsink_kernel(const __grid_constant__ BwdPrepParams p)
{
    __shared__ float red[8];
    const int h = blockIdx.x;
    const float sink = p.sinks[h];
    float acc = 0.f;
    const int n = p.B * p.Tq;
    for (int i = threadIdx.x; i < n; i += 256) {
        const int b = i / p.Tq, t = i % p.Tq;
        const int64_t row = ((int64_t)b * p.H + h) * p.Tq + t;
        const float l = p.lse[row];
        if (l != -INFINITY) acc += expf(sink - l) * p.delta[row];
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.f;
        for (int w = 0; w < 8; ++w) s += red[w];
        p.dsinks[h] = -s;
    }
}

// Row-split dK / dV: sum the fp32 partials of the splits in split order, scale dK, write bf16.
template <int D, int DV>
__global__ void __launch_bounds__(256) bwd_reduce_kernel(const __grid_constant__ BwdParams p)
{
    constexpr int W = D + DV;
    const int64_t x = (int64_t)blockIdx.x * 256 + threadIdx.x;      // one thread per 4 elements
    const int64_t rows = (int64_t)p.B * p.Hkv * p.Tk;
    if (x >= rows * (W / 4)) return;
    const int64_t row = x / (W / 4);
    const int e = (int)(x % (W / 4)) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < p.rsplit; ++s) {
        const float4 v = *reinterpret_cast<const float4 *>(p.dkv_part + ((int64_t)s * rows + row) * W + e);
        acc.x += v.x, acc.y += v.y, acc.z += v.z, acc.w += v.w;
    }
    const int kj = (int)(row % p.Tk), kvh = (int)((row / p.Tk) % p.Hkv), b = (int)(row / ((int64_t)p.Tk * p.Hkv));
    __nv_bfloat16 *dst;
    float f = 1.f;
    if (e >= p.dk_cols && e < D) return;      // MLA rope columns: summed over heads elsewhere
    if (e < D) {
        dst = p.dk + (int64_t)b * p.dks[0] + (int64_t)kvh * p.dks[1] + (int64_t)kj * p.dks[2] + e;
        f = p.scale;
    } else {
        dst = p.dv + (int64_t)b * p.dvs[0] + (int64_t)kvh * p.dvs[1] + (int64_t)kj * p.dvs[2] + (e - D);
    }
    *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16(acc.x * f, acc.y * f), pack_bf16(acc.z * f, acc.w * f));
}

// MLA: dk_rope[b, kj] = scale * sum over row splits and heads of the per-head rope columns
// of dK, in a fixed order; one thread per 4 columns.
__global__ void __launch_bounds__(256) bwd_rope_reduce_kernel(const __grid_constant__ BwdParams p)
{
    const int dr = p.D - p.dk_cols;
    const int64_t x = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const int64_t rows = (int64_t)p.B * p.Tk;
    if (x >= rows * (dr / 4)) return;
    const int64_t row = x / (dr / 4);
    const int e = (int)(x % (dr / 4)) * 4;
    const int kj = (int)(row % p.Tk), b = (int)(row / p.Tk);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < p.rsplit; ++s)
        for (int h = 0; h < p.Hkv; ++h) {
            const float4 v =
                *reinterpret_cast<const float4 *>(p.dkr_part + ((((int64_t)s * p.B + b) * p.Hkv + h) * p.Tk + kj) * dr + e);
            acc.x += v.x, acc.y += v.y, acc.z += v.z, acc.w += v.w;
        }
    __nv_bfloat16 *dst = p.dk2 + (int64_t)b * p.dk2s[0] + (int64_t)kj * p.dk2s[1] + e;
    *reinterpret_cast<uint2 *>(dst) =
        make_uint2(pack_bf16(acc.x * p.scale, acc.y * p.scale), pack_bf16(acc.z * p.scale, acc.w * p.scale));
}

template <int D, int DV, int BR, int NH>
cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t s)
{
    cudaError_t e;
    {
        using L = DkdvLayout<D, DV, BR, NH>;
        auto kern = bwd_dkdv_kernel<D, DV, BR, NH>;
        // at least 116 KB so one CTA holds an SM: each allocates all 512 TMEM columns
        const int bytes = L::BYTES > 118784 ? L::BYTES : 118784;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess) return e;
        const int grid = p.B * p.Hkv * ((p.Tk + BK - 1) / BK) * p.rsplit;
        if (grid > 0) kern<<<grid, DKDV_THREADS, bytes, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (p.rsplit > 1 && p.Tk > 0) {
        const int64_t n = (int64_t)p.B * p.Hkv * p.Tk * ((D + DV) / 4);
        bwd_reduce_kernel<D, DV><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (p.mla && p.Tk > 0 && p.dk_cols < D) {
        const int64_t n = (int64_t)p.B * p.Tk * ((D - p.dk_cols) / 4);
        bwd_rope_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        auto kern = bwd_dq_kernel<D, DV>;
        const int bytes = DqLayout<D, DV>::BYTES > 118784 ? DqLayout<D, DV>::BYTES : 118784;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess) return e;
        const int grid = p.B * p.Hkv * ((p.G * p.Tq + BQ - 1) / BQ);
        kern<<<grid, BW_THREADS, bytes, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

bool bwd_supported(int d, int dv) { return (d == 64 && dv == 64) || (d == 128 && dv == 128) || (d == 192 && dv == 128); }

// fold rows per dK/dV tile: 128, or 64 where TMEM needs the room (d 192)
int bwd_tile_rows(int d, int dv) { return d + dv + 2 * 128 <= 512 ? 128 : 64; }

cudaError_t launch_bwd_prep(const BwdPrepParams &p, cudaStream_t s)
{
    const int64_t rows = (int64_t)p.B * p.H * p.Tq;
    if (rows == 0) return cudaSuccess;
    const int64_t per_cta = 8 * PREP_U * (p.Dv >= 256 ? 1 : 256 / p.Dv);   // rows per CTA, as in the kernel
    bwd_prep_kernel<<<(unsigned)((rows + per_cta - 1) / per_cta), 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !p.sinks) return e;
    bwd_dsink_kernel<<<p.H, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdParams &p, cudaStream_t s)
{
    if (p.D == 64 && p.Dv == 64) return launch_bwd_t<64, 64, 128, 2>(p, s);
    if (p.D == 128 && p.Dv == 128) return launch_bwd_t<128, 128, 128, 2>(p, s);
    if (p.D == 192 && p.Dv == 128) return launch_bwd_t<192, 128, 64, 1>(p, s);
    return cudaErrorInvalidValue;
}

int bwd_dkdv_smem_bytes(int d, int dv)
{
    if (d == 64) return DkdvLayout<64, 64, 128, 2>::BYTES;
    if (d == 128) return DkdvLayout<128, 128, 128, 2>::BYTES;
    return DkdvLayout<192, 128, 64, 1>::BYTES;
}

int bwd_dq_smem_bytes(int d, int dv)
{
    if (d == 64) return DqLayout<64, 64>::BYTES;
    if (d == 128) return DqLayout<128, 128>::BYTES;
    return DqLayout<192, 128>::BYTES;
}

}  // namespace arc
