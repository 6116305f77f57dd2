// attn_tc.cu -- fused attention forward on tcgen05 tensor cores (sm_100a):
// dense / GQA-folded / MLA, bf16 in, fp32 accumulate, O and LSE out.
//
// One CTA owns a tile of 128 query rows of one (batch, kv head) group and one
// slice of d_v columns.  The GQA fold is pure index math: the g*Tq query rows
// that share kv head `kv` are the contiguous rows kv*g*Tq .. of q viewed as
// [B, H*Tq, D] ("ArcFlash ... rung 0", Fold section), so a tile may straddle
// two query heads and every row computes its own position t = r mod Tq for the
// causal mask.  Query rows are independent softmaxes, so tiles never exchange
// anything (same page, Tile section).
//
// Warp roles (256 threads):
//   warp 0      TMA producer: Q once, then K and V tiles in 64-column chunks
//               through a ring of shared-memory stages
//   warp 1      TMEM owner and MMA issuer (one elected lane):
//                 S[buf] = Q K^T      (M=128, N=128, K-major A and B)
//                 O     += P V        (M=128, N=d_v slice, V read MN-major)
//   warps 4-7   softmax: one thread per query row; read S from TMEM, mask,
//               online max / sum in log2 units, write P (bf16, two per 32-bit
//               column) back over the S columns it came from, rescale O in
//               TMEM when the running max grows by more than 2^8, epilogue.
// TMEM (512 columns): O slice at columns [0, DVS), S/P double buffer at 256, 384.
// P is the TMEM A operand of O += P V, so P never touches shared memory; S of
// tile j+2 reuses the buffer only after O += P_j V_j, which the tensor core
// executes in issue order.
// Every wait is bounded; a wait that runs out reports through p.status.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace arc {
namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int CHUNK = BM * 128;     // bytes of one [128 rows x 64 bf16] swizzled chunk
constexpr int NTHREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int S_COL = 256;
constexpr int MAX_STAGES = 12;
constexpr int SMEM_LIMIT = 232448;  // 227 KB opt-in maximum per block
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

struct Bars {
    uint64_t q_full;
    uint64_t s_full[2];
    uint64_t p_full;
    uint64_t o_done;
    uint64_t drain;
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint32_t tmem_base;
};

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

template <int DQK, int DVS, bool MLA>
__global__ void __launch_bounds__(NTHREADS, 1) tc_attn_kernel(const __grid_constant__ TcParams p)
{
    constexpr int KC = DQK / 64;  // 64-column chunks of a Q / K row
    constexpr int VC = DVS / 64;  // 64-column chunks of this CTA's V slice
    static_assert(DQK % 64 == 0 && DVS % 64 == 0 && DVS <= 256, "tile shape");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem<1024>(smem_raw);
    uint8_t *sQ = smem;
    uint8_t *sRing = sQ + KC * CHUNK;
    const int R = p.stages;
    Bars *bars = reinterpret_cast<Bars *>(sRing + R * CHUNK);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- which tile this CTA owns
    const int groups = p.B * p.Hkv * p.n_slices;
    const int rank = blockIdx.x / groups;
    const int rest = blockIdx.x % groups;
    const int slice = rest % p.n_slices;
    const int kv = (rest / p.n_slices) % p.Hkv;
    const int b = rest / (p.n_slices * p.Hkv);
    const int tile = rank < 1024 ? (int)p.tile_order[rank] : rank;
    const int rows_in_group = p.G * p.Tq;
    const int r0 = tile * BM;
    const int dv0 = slice * DVS;
    int nt;
    {
        const int r_last = min(r0 + BM, rows_in_group) - 1;
        const int t_max = (r0 / p.Tq != r_last / p.Tq) ? p.Tq - 1 : r_last % p.Tq;
        const int kv_last = p.causal ? min(p.Tk - 1, t_max + p.Tk - p.Tq) : p.Tk - 1;
        nt = kv_last < 0 ? 0 : kv_last / BN + 1;
    }

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int i = 0; i < 2; ++i) mbar_init(&bars->s_full[i], 1);
        mbar_init(&bars->p_full, 128);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        for (int i = 0; i < R; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], 1);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // =============================== TMA producer
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&p.tm_q);
            tma_prefetch_desc(&p.tm_k);
            tma_prefetch_desc(&p.tm_v);
            const int qrow = kv * rows_in_group + r0;  // row in the [H*Tq] view
            mbar_arrive_expect_tx(&bars->q_full, KC * CHUNK);
            for (int c = 0; c < KC; ++c) {
                if (!MLA || c < p.kc_first)
                    tma_load_3d(sQ + c * CHUNK, &p.tm_q, &bars->q_full, c * 64, qrow, b);
                else
                    tma_load_3d(sQ + c * CHUNK, &p.tm_q2, &bars->q_full, (c - p.kc_first) * 64, qrow, b);
            }
            int stage = 0;
            uint32_t ephase = 0;
            int total = 0;  // chunk loads issued so far (stage of load i is i % R)
            bool ok = true;
            auto acquire = [&]() -> bool {
                if (!mbar_wait(&bars->empty[stage], ephase ^ 1u)) return false;
                mbar_arrive_expect_tx(&bars->full[stage], CHUNK);
                ++total;
                return true;
            };
            auto advance = [&]() {
                if (++stage == R) {
                    stage = 0;
                    ephase ^= 1u;
                }
            };
            auto load_k = [&](int j) -> bool {
                for (int c = 0; c < KC; ++c) {
                    if (!acquire()) return false;
                    uint8_t *dst = sRing + stage * CHUNK;
                    if (!MLA || c < p.kc_first)
                        tma_load_4d(dst, &p.tm_k, &bars->full[stage], c * 64, j * BN, kv, b);
                    else
                        tma_load_3d(dst, &p.tm_k2, &bars->full[stage], (c - p.kc_first) * 64, j * BN, b);
                    advance();
                }
                return true;
            };
            auto load_v = [&](int j) -> bool {
                for (int c = 0; c < VC; ++c) {
                    if (!acquire()) return false;
                    tma_load_4d(sRing + stage * CHUNK, &p.tm_v, &bars->full[stage], dv0 + c * 64, j * BN, kv, b);
                    advance();
                }
                return true;
            };
            ok = load_k(0);
            for (int j = 0; ok && j < nt; ++j) {
                if (j + 1 < nt) ok = load_k(j + 1);
                if (ok) ok = load_v(j);
            }
            if (!ok) report(p.status, ST_TIMEOUT_LOAD);
            // Drain: every copy this thread issued has landed before the CTA exits.
            for (int s = 0; s < R && s < total; ++s) {
                const int loads = (total - s + R - 1) / R;  // loads that went to stage s
                mbar_wait(&bars->full[s], (uint32_t)((loads - 1) & 1));
            }
            mbar_wait(&bars->q_full, 0);
        }
    } else if (warp == 1) {
        // =============================== MMA issuer
        // Kept lean on purpose: one thread issues every MMA, so descriptors are
        // precomputed and advanced by constants, four K steps go out per issue block,
        // and nothing here touches local memory.
        if (lane == 0 && nt > 0) {
            constexpr uint32_t kChunkUnits = CHUNK >> 4;     // descriptor units per ring stage
            const uint32_t idesc_s = idesc_bf16(BM, BN, false, false);
            const uint64_t qd0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t kd0 = sdesc_sw128(smem_u32(sRing), 16, 1024);
            const uint64_t vd0 = sdesc_sw128(smem_u32(sRing), CHUNK, 1024);
            int stage = 0;
            uint32_t fphase = 0;
            bool ok = mbar_wait(&bars->q_full, 0);
            tc_fence_after();
            auto advance = [&]() {
                if (++stage == R) {
                    stage = 0;
                    fphase ^= 1u;
                }
            };
            auto issue_s = [&](int j) -> bool {
                const uint32_t d = tmem + S_COL + (j & 1) * BN;
#pragma unroll 1
                for (int c = 0; c < KC; ++c) {
                    if (!mbar_wait(&bars->full[stage], fphase)) return false;
                    tc_fence_after();
                    umma_ss_k64(d, qd0 + (uint64_t)(c * kChunkUnits), kd0 + (uint64_t)(stage * kChunkUnits), idesc_s,
                                c > 0);
                    umma_commit(&bars->empty[stage]);
                    advance();
                }
                umma_commit(&bars->s_full[j & 1]);
                return true;
            };
            auto issue_pv = [&](int j) -> bool {
                if (!mbar_wait(&bars->p_full, (uint32_t)(j & 1))) return false;
                const int s0 = stage;
#pragma unroll 1
                for (int c = 0; c < VC; ++c) {
                    if (!mbar_wait(&bars->full[stage], fphase)) return false;
                    advance();
                }
                tc_fence_after();
                const uint32_t p_tm = tmem + S_COL + (j & 1) * BN;
                // V chunks sit in stages s0.. (wrapping at R): at most two contiguous runs.
                const int n1 = (s0 + VC <= R) ? VC : R - s0;
                const uint32_t idesc1 = idesc_bf16(BM, 64 * n1, false, true);
                const uint64_t b1 = vd0 + (uint64_t)(s0 * kChunkUnits);
                const uint32_t acc = j > 0;
#pragma unroll
                for (int k4 = 0; k4 < BN / 64; ++k4)
                    umma_ts_k64(tmem, p_tm + k4 * 32, b1 + (uint64_t)(k4 * 512), 128, idesc1, acc | k4);
                if (n1 < VC) {
                    const uint32_t idesc2 = idesc_bf16(BM, 64 * (VC - n1), false, true);
#pragma unroll
                    for (int k4 = 0; k4 < BN / 64; ++k4)
                        umma_ts_k64(tmem + n1 * 64, p_tm + k4 * 32, vd0 + (uint64_t)(k4 * 512), 128, idesc2, acc | k4);
                }
#pragma unroll 1
                for (int c = 0; c < VC; ++c) umma_commit(&bars->empty[(s0 + c) % R]);
                umma_commit(&bars->o_done);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 0; ok && j < nt; ++j) {
                if (j + 1 < nt) ok = issue_s(j + 1);
                if (ok) ok = issue_pv(j);
            }
            if (!ok) report(p.status, ST_TIMEOUT_MMA);
            // Drain: all MMAs issued by this thread complete before TMEM is freed.
            umma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0);
        }
    } else if (warp >= 4) {
        // =============================== softmax, correction, epilogue
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const int R_ = r0 + r;
        const bool row_ok = R_ < rows_in_group;
        const int t = R_ % p.Tq;
        const int h = kv * p.G + R_ / p.Tq;
        const int last = p.causal ? min(p.Tk - 1, t + p.Tk - p.Tq) : p.Tk - 1;
        const float sl2 = p.scale_log2;
        float m_use = -INFINITY, l = 0.f;
        bool ok = true;

        for (int j = 0; j < nt; ++j) {
            const int buf = j & 1;
            const uint32_t s_tmem = tmem + lane_off + S_COL + buf * BN;
            ok = warp_all(mbar_wait(&bars->s_full[buf], (uint32_t)((j >> 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[BN];
#pragma unroll
            for (int i = 0; i < BN / 32; ++i)
                tmem_ld32(s_tmem + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * i]));
            tmem_wait_ld();

            const int kbase = j * BN;
            if (kbase + BN - 1 > last) {
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (kbase + i > last) sv[i] = __float_as_uint(-INFINITY);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < BN; ++i) mx = fmaxf(mx, __uint_as_float(sv[i]));
            mx *= sl2;
            const bool need = mx > m_use + RESCALE_THRESHOLD;
            float alpha = 1.f;
            if (need) {
                alpha = (m_use == -INFINITY) ? 0.f : fast_exp2(m_use - mx);
                m_use = mx;
            }
            const float msafe = (m_use == -INFINITY) ? 0.f : m_use;
            float rowsum = 0.f;
            uint32_t pk0[32], pk1[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * i]), sl2, -msafe));
                const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * i + 1]), sl2, -msafe));
                rowsum += p0 + p1;
                pk0[i] = pack_bf16(p0, p1);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float p0 = fast_exp2(fmaf(__uint_as_float(sv[64 + 2 * i]), sl2, -msafe));
                const float p1 = fast_exp2(fmaf(__uint_as_float(sv[64 + 2 * i + 1]), sl2, -msafe));
                rowsum += p0 + p1;
                pk1[i] = pack_bf16(p0, p1);
            }
            l = l * alpha + rowsum;
            // P (bf16 pairs) over the first half of the S columns it came from.
            tmem_st32(s_tmem, pk0);
            tmem_st32(s_tmem + 32, pk1);

            // O += P(j-1) V(j-1) must be complete before O is rescaled; waiting on
            // every tile keeps this thread's view of o_done in step with its phases.
            if (j > 0) {
                ok = warp_all(mbar_wait(&bars->o_done, (uint32_t)((j - 1) & 1)));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                    for (int c = 0; c < DVS / 32; ++c) {
                        uint32_t ov[32];
                        tmem_ld32(tmem + lane_off + 32 * c, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st32(tmem + lane_off + 32 * c, ov);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full);
        }
        if (ok && nt > 0) {
            ok = warp_all(mbar_wait(&bars->o_done, (uint32_t)((nt - 1) & 1)));
            tc_fence_after();
        }
        if (!ok) report(p.status, ST_TIMEOUT_SOFTMAX);

        // ---- final normalisation; the sink joins the denominator only
        float fac, lse;
        if (p.sinks) {
            const float sg = row_ok ? p.sinks[h] * LOG2E : 0.f;  // padding rows may lie past the last head
            const float mf = fmaxf(m_use, sg);
            const float a = (m_use == -INFINITY) ? 0.f : exp2f(m_use - mf);
            const float lf = l * a + exp2f(sg - mf);
            fac = a / lf;
            lse = (mf + log2f(lf)) * LN2;
        } else {
            fac = l > 0.f ? 1.f / l : 0.f;
            lse = l > 0.f ? (m_use + log2f(l)) * LN2 : -INFINITY;
        }
        __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(p.o) + (int64_t)b * p.os[0] + (int64_t)h * p.os[1] +
                              (int64_t)t * p.os[2] + dv0;
#pragma unroll 1
        for (int c = 0; c < DVS / 32; ++c) {
            uint32_t ov[32];
            if (nt > 0 && ok) {
                tmem_ld32(tmem + lane_off + 32 * c, ov);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = 0u;
            }
            if (row_ok) {
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16(__uint_as_float(ov[2 * i]) * fac, __uint_as_float(ov[2 * i + 1]) * fac);
                uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
        if (row_ok && slice == 0) p.lse[((int64_t)b * p.H + h) * p.Tq + t] = lse;
    }

    // Each warp arrives whole (a role branch may have left lanes behind, e.g. the MMA
    // issuer's lane 0), so the barrier below holds until every warp is done with TMEM.
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Two query tiles per CTA (d_v <= 128).  Tiles A and B are 128 consecutive fold
// rows each of the same (batch, kv head) group, so every K/V tile the producer
// brings in feeds both: half the shared-memory and L2 traffic per FLOP of the
// one-tile kernel.  TMEM: O_A [0,128), S/P_A [128,256), O_B [256,384),
// S/P_B [384,512).  MMA order per KV tile j (steady state):
//     O_A += P_A(j) V(j),  S_A(j+1),  O_B += P_B(j) V(j),  S_B(j+1)
// so softmax A(j+1) overlaps the B-side MMAs and softmax B(j+1) the A side.
// Softmax warps 2-5 serve tile A, warps 6-9 tile B (a warp reads TMEM lanes
// 32*(warp % 4) .. +31); each loads its whole S row, then writes P over it.
constexpr int NTHREADS2 = 320;  // producer, MMA, two softmax warpgroups

template <int DQK, int DVS, bool MLA>
__global__ void __launch_bounds__(NTHREADS2, 1) tc_attn2_kernel(const __grid_constant__ TcParams p)
{
    constexpr int KC = DQK / 64;
    constexpr int VC = DVS / 64;
    static_assert(DQK % 64 == 0 && DVS % 64 == 0 && DVS <= 128, "tile shape");
    // TMEM columns of tile t: O at 256*t, S/P at 128 + 256*t
#define O_COL(t) (256u * (uint32_t)(t))
#define S_COL2(t) (128u + 256u * (uint32_t)(t))

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem<1024>(smem_raw);
    uint8_t *sQ = smem;                       // [2 tiles][KC chunks]
    uint8_t *sRing = sQ + 2 * KC * CHUNK;
    const int R = p.stages;
    struct Bars2 {
        uint64_t q_full;
        uint64_t s_full[2];
        uint64_t p_full[2];
        uint64_t o_done[2];
        uint64_t drain;
        uint64_t full[MAX_STAGES];
        uint64_t empty[MAX_STAGES];
        uint32_t tmem_base;
    };
    Bars2 *bars = reinterpret_cast<Bars2 *>(sRing + R * CHUNK);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int groups = p.B * p.Hkv;
    const int rank = blockIdx.x / groups;
    const int rest = blockIdx.x % groups;
    const int kv = rest % p.Hkv;
    const int b = rest / p.Hkv;
    const int pair = rank < 1024 ? (int)p.tile_order[rank] : rank;
    const int rows_in_group = p.G * p.Tq;
    const int r0 = pair * 2 * BM;
    int nt;  // KV tiles covering both query tiles
    {
        const int r_last = min(r0 + 2 * BM, rows_in_group) - 1;
        const int t_max = (r0 / p.Tq != r_last / p.Tq) ? p.Tq - 1 : r_last % p.Tq;
        const int kv_last = p.causal ? min(p.Tk - 1, t_max + p.Tk - p.Tq) : p.Tk - 1;
        nt = kv_last < 0 ? 0 : kv_last / BN + 1;
    }

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 128);
            mbar_init(&bars->o_done[i], 1);
        }
        mbar_init(&bars->drain, 1);
        for (int i = 0; i < R; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], 1);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // =============================== TMA producer: Q_A, Q_B, then K(0), V(0), K(1), V(1), ...
        // A barrier round trip costs the issuing thread a few hundred clocks, so the
        // KC + VC chunks of a tile are handled by that many lanes at once: each lane
        // waits for its own ring slot and issues its own load.
        if (nt > 0) {
            if (lane == 0) {
                tma_prefetch_desc(&p.tm_q);
                tma_prefetch_desc(&p.tm_k);
                tma_prefetch_desc(&p.tm_v);
                const int qrow = kv * rows_in_group + r0;
                mbar_arrive_expect_tx(&bars->q_full, 2 * KC * CHUNK);
                for (int t = 0; t < 2; ++t)
                    for (int c = 0; c < KC; ++c) {
                        uint8_t *dst = sQ + (t * KC + c) * CHUNK;
                        if (!MLA || c < p.kc_first)
                            tma_load_3d(dst, &p.tm_q, &bars->q_full, c * 64, qrow + t * BM, b);
                        else
                            tma_load_3d(dst, &p.tm_q2, &bars->q_full, (c - p.kc_first) * 64, qrow + t * BM, b);
                    }
            }
            __syncwarp();
            constexpr int PER = KC + VC;   // chunks per KV tile (<= 32: one lane each)
            static_assert(PER <= 32, "one lane per chunk of a tile");
            const int total = nt * PER;
            bool ok = true;
            for (int j = 0; ok && j < nt; ++j) {
                bool mine = true;
                if (lane < PER) {
                    const int n = j * PER + lane;                 // chunk index in the load sequence
                    const int st = n % R;
                    mine = mbar_wait(&bars->empty[st], (uint32_t)(((n / R) & 1) ^ 1));
                    if (mine) {
                        mbar_arrive_expect_tx(&bars->full[st], CHUNK);
                        uint8_t *dst = sRing + st * CHUNK;
                        if (lane < KC) {
                            const int c = lane;
                            if (!MLA || c < p.kc_first)
                                tma_load_4d(dst, &p.tm_k, &bars->full[st], c * 64, j * BN, kv, b);
                            else
                                tma_load_3d(dst, &p.tm_k2, &bars->full[st], (c - p.kc_first) * 64, j * BN, b);
                        } else {
                            tma_load_4d(dst, &p.tm_v, &bars->full[st], (lane - KC) * 64, j * BN, kv, b);
                        }
                    }
                }
                ok = __all_sync(0xffffffffu, mine);
            }
            if (lane == 0) {
                if (!ok) report(p.status, ST_TIMEOUT_LOAD);
                for (int s = 0; s < R && s < total; ++s) {
                    const int loads = (total - s + R - 1) / R;
                    mbar_wait(&bars->full[s], (uint32_t)((loads - 1) & 1));
                }
                mbar_wait(&bars->q_full, 0);
            }
        }
    } else if (warp == 1) {
        // =============================== MMA issuer
        if (lane == 0 && nt > 0) {
            constexpr uint32_t kChunkUnits = CHUNK >> 4;
            const uint32_t idesc_s = idesc_bf16(BM, BN, false, false);
            const uint64_t qd0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t kd0 = sdesc_sw128(smem_u32(sRing), 16, 1024);
            const uint64_t vd0 = sdesc_sw128(smem_u32(sRing), CHUNK, 1024);
            int stage = 0;
            uint32_t fphase = 0;
            bool ok = mbar_wait(&bars->q_full, 0);
            tc_fence_after();
            auto advance = [&]() {
                if (++stage == R) {
                    stage = 0;
                    fphase ^= 1u;
                }
            };
            // First use of the next KC (or VC) ring stages: wait for each and return the first.
            auto take = [&](int n, int &first) -> bool {
                first = stage;
                for (int c = 0; c < n; ++c) {
                    if (!mbar_wait(&bars->full[stage], fphase)) return false;
                    advance();
                }
                tc_fence_after();
                return true;
            };
            auto issue_s = [&](int t, int k0) {
                const uint32_t d = tmem + S_COL2(t);
#pragma unroll
                for (int c = 0; c < KC; ++c)
                    umma_ss_k64(d, qd0 + (uint64_t)((t * KC + c) * kChunkUnits),
                                kd0 + (uint64_t)(((k0 + c) % R) * kChunkUnits), idesc_s, c > 0);
                umma_commit(&bars->s_full[t]);
            };
            auto issue_pv = [&](int t, int j, int v0) {
                const uint32_t p_tm = tmem + S_COL2(t);
                const int n1 = (v0 + VC <= R) ? VC : R - v0;
                const uint32_t idesc1 = idesc_bf16(BM, 64 * n1, false, true);
#pragma unroll
                for (int k4 = 0; k4 < BN / 64; ++k4)
                    umma_ts_k64(tmem + O_COL(t), p_tm + k4 * 32, vd0 + (uint64_t)(v0 * kChunkUnits + k4 * 512), 128,
                                idesc1, (j > 0) | k4);
                if (n1 < VC) {
                    const uint32_t idesc2 = idesc_bf16(BM, 64 * (VC - n1), false, true);
#pragma unroll
                    for (int k4 = 0; k4 < BN / 64; ++k4)
                        umma_ts_k64(tmem + O_COL(t) + n1 * 64, p_tm + k4 * 32, vd0 + (uint64_t)(k4 * 512), 128, idesc2,
                                    (j > 0) | k4);
                }
                umma_commit(&bars->o_done[t]);
            };
            auto release = [&](int first, int n) {
                for (int c = 0; c < n; ++c) umma_commit(&bars->empty[(first + c) % R]);
            };
            int k0 = 0, v0 = 0;
            if (ok) ok = take(KC, k0);
            if (ok) {
                issue_s(0, k0);
                issue_s(1, k0);
                release(k0, KC);
            }
            for (int j = 0; ok && j < nt; ++j) {
                if (!(ok = take(VC, v0))) break;
                if (!(ok = mbar_wait(&bars->p_full[0], (uint32_t)(j & 1)))) break;
                tc_fence_after();
                issue_pv(0, j, v0);
                const bool more = j + 1 < nt;
                if (more) {
                    if (!(ok = take(KC, k0))) break;
                    issue_s(0, k0);
                }
                if (!(ok = mbar_wait(&bars->p_full[1], (uint32_t)(j & 1)))) break;
                tc_fence_after();
                issue_pv(1, j, v0);
                release(v0, VC);
                if (more) {
                    issue_s(1, k0);
                    release(k0, KC);
                }
            }
            if (!ok) report(p.status, ST_TIMEOUT_MMA);
            umma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0);
        }
    } else {
        // =============================== softmax (warps 2-5: tile A, 6-9: tile B) and epilogue
        const int t = (warp - 2) >> 2;
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const int R_ = r0 + t * BM + r;
        const bool row_ok = R_ < rows_in_group;
        const int tpos = R_ % p.Tq;
        const int h = kv * p.G + R_ / p.Tq;
        const int last = p.causal ? min(p.Tk - 1, tpos + p.Tk - p.Tq) : p.Tk - 1;
        const float sl2 = p.scale_log2;
        const uint32_t s_tmem = tmem + lane_off + S_COL2(t);
        const uint32_t o_tmem = tmem + lane_off + O_COL(t);
        float m_use = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            ok = warp_all(mbar_wait(&bars->s_full[t], (uint32_t)(j & 1)));
            if (!ok) break;
            tc_fence_after();
            const int kbase = j * BN;
            // All of S in one go (four loads, one wait), then P written over it in place.
            uint32_t sv[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
                tmem_ld32(s_tmem + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * c]));
            tmem_wait_ld();
            if (kbase + BN - 1 > last) {
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (kbase + i > last) sv[i] = __float_as_uint(-INFINITY);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < BN; ++i) mx = fmaxf(mx, __uint_as_float(sv[i]));
            mx *= sl2;
            const bool need = mx > m_use + RESCALE_THRESHOLD;
            float alpha = 1.f;
            if (need) {
                alpha = (m_use == -INFINITY) ? 0.f : fast_exp2(m_use - mx);
                m_use = mx;
            }
            const float msafe = (m_use == -INFINITY) ? 0.f : m_use;
            float rowsum = 0.f;
#pragma unroll
            for (int c = 0; c < BN / 8; ++c) {
                uint32_t pk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float p0 = fast_exp2(fmaf(__uint_as_float(sv[8 * c + 2 * i]), sl2, -msafe));
                    const float p1 = fast_exp2(fmaf(__uint_as_float(sv[8 * c + 2 * i + 1]), sl2, -msafe));
                    rowsum += p0 + p1;
                    pk[i] = pack_bf16(p0, p1);
                }
                tmem_st4(s_tmem + 4 * c, pk[0], pk[1], pk[2], pk[3]);
            }
            l = l * alpha + rowsum;
            if (j > 0) {
                ok = warp_all(mbar_wait(&bars->o_done[t], (uint32_t)((j - 1) & 1)));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                    for (int c = 0; c < DVS / 32; ++c) {
                        uint32_t ov[32];
                        tmem_ld32(o_tmem + 32 * c, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st32(o_tmem + 32 * c, ov);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[t]);
        }
        if (ok && nt > 0) {
            ok = warp_all(mbar_wait(&bars->o_done[t], (uint32_t)((nt - 1) & 1)));
            tc_fence_after();
        }
        if (!ok) report(p.status, ST_TIMEOUT_SOFTMAX);
        float fac, lse;
        if (p.sinks) {
            const float sg = row_ok ? p.sinks[h] * LOG2E : 0.f;
            const float mf = fmaxf(m_use, sg);
            const float a = (m_use == -INFINITY) ? 0.f : exp2f(m_use - mf);
            const float lf = l * a + exp2f(sg - mf);
            fac = a / lf;
            lse = (mf + log2f(lf)) * LN2;
        } else {
            fac = l > 0.f ? 1.f / l : 0.f;
            lse = l > 0.f ? (m_use + log2f(l)) * LN2 : -INFINITY;
        }
        __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(p.o) + (int64_t)b * p.os[0] + (int64_t)h * p.os[1] +
                              (int64_t)tpos * p.os[2];
#pragma unroll 1
        for (int c = 0; c < DVS / 32; ++c) {
            uint32_t ov[32];
            if (nt > 0 && ok) {
                tmem_ld32(o_tmem + 32 * c, ov);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = 0u;
            }
            if (row_ok) {
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16(__uint_as_float(ov[2 * i]) * fac, __uint_as_float(ov[2 * i + 1]) * fac);
                uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
        if (row_ok) p.lse[((int64_t)b * p.H + h) * p.Tq + tpos] = lse;
    }

    // Each warp arrives whole (a role branch may have left lanes behind, e.g. the MMA
    // issuer's lane 0), so the barrier below holds until every warp is done with TMEM.
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

#undef O_COL
#undef S_COL2

template <int DQK, int DVS, bool MLA>
cudaError_t launch_two(const TcParams &p, int grid, cudaStream_t s)
{
    const int smem = tc2_smem_bytes(DQK, p.stages);
    auto kern = tc_attn2_kernel<DQK, DVS, MLA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, NTHREADS2, smem, s>>>(p);
    return cudaGetLastError();
}

template <int DQK, int DVS, bool MLA>
cudaError_t launch_one(const TcParams &p, int grid, cudaStream_t s)
{
    const int smem = tc_smem_bytes(DQK, p.stages);
    auto kern = tc_attn_kernel<DQK, DVS, MLA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, NTHREADS, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

int tc2_smem_bytes(int dqk, int stages) { return 1024 + (2 * (dqk / 64) + stages) * CHUNK + 512; }

int tc2_max_stages(int dqk)
{
    int st = (SMEM_LIMIT - 1024 - 512 - 2 * (dqk / 64) * CHUNK) / CHUNK;
    return st < MAX_STAGES ? st : MAX_STAGES;
}

cudaError_t launch_tc_attn2(const TcParams &p, int dqk, int dvs, bool mla, int grid, cudaStream_t s)
{
#define ARC_TC2_CASE(Q, V, M) \
    if (dqk == Q && dvs == V && mla == M) return launch_two<Q, V, M>(p, grid, s);
    ARC_TC2_CASE(64, 64, false)
    ARC_TC2_CASE(128, 64, false)
    ARC_TC2_CASE(128, 128, false)
    ARC_TC2_CASE(192, 128, false)
    ARC_TC2_CASE(256, 128, false)
    ARC_TC2_CASE(128, 128, true)
    ARC_TC2_CASE(192, 128, true)
    ARC_TC2_CASE(192, 64, true)
    ARC_TC2_CASE(256, 128, true)
#undef ARC_TC2_CASE
    return cudaErrorInvalidValue;
}

int tc_smem_bytes(int dqk, int stages) { return 1024 + (dqk / 64 + stages) * CHUNK + (int)sizeof(Bars); }

int tc_max_stages(int dqk)
{
    int st = (SMEM_LIMIT - 1024 - (int)sizeof(Bars) - (dqk / 64) * CHUNK) / CHUNK;
    return st < MAX_STAGES ? st : MAX_STAGES;
}

cudaError_t launch_tc_attn(const TcParams &p, int dqk, int dvs, bool mla, int grid, cudaStream_t s)
{
#define ARC_TC_CASE(Q, V, M) \
    if (dqk == Q && dvs == V && mla == M) return launch_one<Q, V, M>(p, grid, s);
    ARC_TC_CASE(64, 64, false)
    ARC_TC_CASE(128, 64, false)
    ARC_TC_CASE(128, 128, false)
    ARC_TC_CASE(192, 128, false)
    ARC_TC_CASE(256, 128, false)
    ARC_TC_CASE(256, 256, false)
    ARC_TC_CASE(512, 256, false)
    ARC_TC_CASE(512, 128, false)
    ARC_TC_CASE(128, 128, true)
    ARC_TC_CASE(192, 128, true)
    ARC_TC_CASE(192, 64, true)
    ARC_TC_CASE(256, 128, true)
    ARC_TC_CASE(256, 256, true)
#undef ARC_TC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace arc
