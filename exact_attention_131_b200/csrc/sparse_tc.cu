// sparse_tc.cu -- sparse (top-k) attention forward on tcgen05 tensor cores.
//
// "TensorRT-LLM: FlashMLA without -rdc", timing paragraph: every query token
// attends, with all of its heads, to its own list of top-k rows of a shared
// KV pool (d_qk 512, 64 heads, 2176 indices per query).  All heads of a token
// read the same gathered rows, so one CTA owns one token and up to 64 heads:
// the MMA is M = 64 rows (heads) tall.
//
// Data path per CTA
//   warps 0-3   Q rows once, straight into tensor memory (each warp its own
//               lane quadrant); then the top-k rows in tiles of 64 keys, 16-byte
//               cp.async per lane (a warp reads 512 contiguous bytes of one pool
//               row), written into the 128-byte-swizzled K-major layout the
//               tensor core reads; an index outside [0, Skv) writes zeros and
//               clears its bit in the tile's validity mask.  A tile's 64 indices
//               are read once per warp and the next tile's are fetched while this
//               tile's rows are in flight.  Three tile buffers rotate.
//   warp 8      TMEM owner and MMA issuer:
//                 S[buf] = Q K^T       M=64, N=64 keys,  A = Q from TMEM, B K-major
//                 O     += P V         M=64, N<=256,     A = P, V MN-major (shared memory)
//               When V is the latent (no separate V) the same gathered tile
//               serves as K and V, so each row crosses L2 once.
//   warps 4-7   softmax: two threads per head row, each holding 32 of the
//               tile's 64 scores; P (bf16) goes to shared memory.
// Holding Q in tensor memory (S reads it there as a TS-form A operand) frees the
// 64 KB it would take in shared memory for a third tile buffer, so the gather of a
// tile no longer waits for the P V of the tile two before it.  At d 512 the tensor
// pipe is then busy for about 96% of a tile: S (32 K=16 steps at M=64, N=64) takes
// about 2,000 cycles and P V (8 steps at N=256) about 1,300.  An M=64 step costs
// about 32 cycles beyond its half-rate arithmetic whatever its operands' source
// (two alternating accumulators did not change it), which bounds this shape.
// TMEM: an M=64 operand or accumulator uses 16 of the 32 lanes of each quadrant
// (rows 16q .. 16q+15 in lanes 32q .. 32q+15, or 32q+16 .. 32q+31 with the lane
// field set to 16).  An A operand read from TMEM must sit in the same lanes as the
// accumulator it feeds, so Q and S share the upper lanes: Q in columns 0..Dqk/2 (two
// bf16 per column), S in columns 256..383 (two buffers).  The lower lanes hold O in
// columns 0..Dv, which never moves; P V therefore takes P from shared memory (O
// fills its half at d_v 512).  All TMEM loads and stores here use the 16-lane
// shapes, which touch only their own half.
// Every wait is bounded and reports through p.status.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace arc {
namespace {

constexpr int SM_ROWS = 64;        // heads per CTA (MMA M)
constexpr int SBN = 64;            // keys per tile
constexpr int SCHUNK = 64 * 128;   // bytes of one [64 rows x 64 bf16] swizzled chunk
constexpr int S_THREADS = 288;     // 9 warps
constexpr int NSTG = 3;            // gathered tile buffers
constexpr float S_LOG2E = 1.4426950408889634f;
constexpr float S_LN2 = 0.6931471805599453f;
constexpr float S_RESCALE = 8.0f;
// TMEM addresses: O at column 0 of the lower 16 lanes of each quadrant; Q and S in
// the upper 16 lanes (lane field 16)
constexpr uint32_t TM_Q = (16u << 16) + 0;
constexpr uint32_t TM_S = (16u << 16) + 256;

struct SparseBars {
    uint64_t q_full;
    uint64_t kv_full[NSTG];
    uint64_t kv_empty[NSTG];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done;
    uint64_t drain;
    uint32_t mask[NSTG][2];  // validity of the 64 slots of each tile buffer
    uint32_t tmem_base;
};

template <int KC, int VC, bool SEPV>
struct SparseLayout {
    static constexpr int TILE_CHUNKS = KC + (SEPV ? VC : 0);
    static constexpr int TILE_BYTES = TILE_CHUNKS * SCHUNK;
    static constexpr int P_BYTES = SCHUNK;  // [64 rows x 64 keys] bf16
    static constexpr int BYTES = 1024 + NSTG * TILE_BYTES + 2 * P_BYTES + (int)sizeof(SparseBars);
};

__device__ __forceinline__ bool warp_all_sparse(bool ok) { return __all_sync(0xffffffffu, ok); }

__device__ __forceinline__ uint32_t swz(int row, int unit) { return (row >> 3) * 1024 + (row & 7) * 128 + ((unit ^ (row & 7)) << 4); }

template <int KC, int VC, bool SEPV>
__global__ void __launch_bounds__(S_THREADS, 1) sparse_tc_kernel(const __grid_constant__ SparseTcParams p)
{
    using L = SparseLayout<KC, VC, SEPV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem<1024>(smem_raw);
    uint8_t *sKV = smem;                              // NSTG tile buffers
    uint8_t *sP = sKV + NSTG * L::TILE_BYTES;         // 2 P buffers
    SparseBars *bars = reinterpret_cast<SparseBars *>(sP + 2 * L::P_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_hgroups = (p.H + SM_ROWS - 1) / SM_ROWS;
    const int sp = blockIdx.x % p.splits;                      // top-k split (decode-shaped calls)
    const int tok = blockIdx.x / (n_hgroups * p.splits);
    const int h0 = ((blockIdx.x / p.splits) % n_hgroups) * SM_ROWS;
    const int s_begin = sp * p.chunk;                          // this CTA's slots: [s_begin, s_begin + cnt)
    const int cnt = max(0, min(p.topk - s_begin, p.chunk));
    const int nt = (cnt + SBN - 1) / SBN;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 128);
        for (int i = 0; i < NSTG; ++i) {
            mbar_init(&bars->kv_full[i], 128);
            mbar_init(&bars->kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 128);
        }
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp < 4) {
        // =============================== gather
        const int32_t *idx_row = p.idx + (int64_t)tok * p.idx_stride + s_begin;
        // Lane i < 16 of warp w holds the index of tile row w + 4i; warp 0 also holds
        // one index per lane for each half of the tile, for the validity mask.
        auto fetch = [&](int j, int32_t &mine, int32_t &m0, int32_t &m1) {
            const int slot = j * SBN + warp + 4 * (lane & 15);
            mine = (lane < 16 && slot < cnt) ? idx_row[slot] : -1;
            if (warp == 0) {
                const int s0 = j * SBN + lane, s1 = s0 + 32;
                m0 = s0 < cnt ? idx_row[s0] : -1;
                m1 = s1 < cnt ? idx_row[s1] : -1;
            }
        };
        // The first tile's indices and every Q load go out together, before anything
        // waits on either: the CTA's start-up is one memory round trip, not several.
        int32_t mine = -1, m0 = -1, m1 = -1;
        if (nt > 0) fetch(0, mine, m0, m1);
        {
            // Q row r = 16 * warp + (lane & 15) into this warp's lane quadrant: half
            // (lane >> 4) of each 64-column group, i.e. 64 consecutive bf16 per store.
            const int r = warp * 16 + (lane & 15), half = lane >> 4;
            const int h = h0 + r;
            const __nv_bfloat16 *qrow = p.q + (int64_t)tok * p.qs[0] + (int64_t)(h < p.H ? h : 0) * p.qs[1];
            const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + TM_Q;   // + upper-lane field
            uint4 qv[KC / 2][8];
#pragma unroll
            for (int c = 0; c < KC / 2; ++c) {
                const uint4 *src = reinterpret_cast<const uint4 *>(qrow + c * 128 + half * 64);
#pragma unroll
                for (int i = 0; i < 8; ++i) qv[c][i] = h < p.H ? src[i] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int c = 0; c < KC / 2; ++c) {
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    w[4 * i] = qv[c][i].x, w[4 * i + 1] = qv[c][i].y, w[4 * i + 2] = qv[c][i].z, w[4 * i + 3] = qv[c][i].w;
                tmem_st16x2_32(taddr + c * 64, w);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->q_full);
        }

        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            const int b = j % NSTG;
            if (j >= NSTG) {
                ok = warp_all_sparse(mbar_wait(&bars->kv_empty[b], (uint32_t)((j / NSTG - 1) & 1)));
                if (!ok) break;
            }
            uint8_t *tile = sKV + b * L::TILE_BYTES;
#pragma unroll 4
            for (int i = 0; i < SBN / 4; ++i) {
                const int r = warp + 4 * i;
                int32_t key = __shfl_sync(0xffffffffu, mine, i);
                const bool valid = key >= 0 && key < p.Skv;
                if (!valid) key = 0;
                const __nv_bfloat16 *krow = p.kv + (int64_t)key * p.kv_stride;
#pragma unroll
                for (int x = lane; x < KC * 8; x += 32) {
                    const int c = x >> 3, u = x & 7;
                    cp_async16(tile + c * SCHUNK + swz(r, u), krow + x * 8, valid ? 16u : 0u);
                }
                if constexpr (SEPV) {
                    const __nv_bfloat16 *vrow = p.v + (int64_t)key * p.v_stride;
#pragma unroll
                    for (int x = lane; x < VC * 8; x += 32) {
                        const int c = x >> 3, u = x & 7;
                        cp_async16(tile + (KC + c) * SCHUNK + swz(r, u), vrow + x * 8, valid ? 16u : 0u);
                    }
                }
            }
            cp_async_commit_group();
            if (warp == 0) {
                const uint32_t b0 = __ballot_sync(0xffffffffu, m0 >= 0 && m0 < p.Skv);
                const uint32_t b1 = __ballot_sync(0xffffffffu, m1 >= 0 && m1 < p.Skv);
                if (lane == 0) {
                    bars->mask[b][0] = b0;
                    bars->mask[b][1] = b1;
                }
            }
            if (j + 1 < nt) fetch(j + 1, mine, m0, m1);  // next tile's indices fly with this tile's rows
            cp_async_wait_all();
            fence_proxy_async_smem();
            mbar_arrive(&bars->kv_full[b]);
        }
        if (!ok) report(p.status, ST_TIMEOUT_LOAD);
    } else if (warp == 8) {
        // =============================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t kChunkUnits = SCHUNK >> 4;
            const uint32_t idesc_s = idesc_bf16(SM_ROWS, SBN, false, false);
            constexpr int NV = VC * 64;                 // O columns
            constexpr int NG = (NV + 255) / 256;        // N groups of <= 256
            const uint64_t kvd0 = sdesc_sw128(smem_u32(sKV), 16, 1024);
            const uint64_t vd0 = sdesc_sw128(smem_u32(sKV), SCHUNK, 1024);
            const uint64_t pd0 = sdesc_sw128(smem_u32(sP), 16, 1024);
            bool ok = mbar_wait(&bars->q_full, 0);
            tc_fence_after();
            auto issue_s = [&](int j) {
                const int b = j % NSTG;
                tc_fence_after();
                const uint32_t d = tmem + TM_S + (j & 1) * SBN;
#pragma unroll
                for (int c = 0; c < KC; ++c)
                    umma_ts_k64(d, tmem + TM_Q + c * 32, kvd0 + (uint64_t)((b * L::TILE_CHUNKS + c) * kChunkUnits), 2,
                                idesc_s, c > 0);
                umma_commit(&bars->s_full[j & 1]);
            };
            auto issue_pv = [&](int j) {
                const int b = j % NSTG;
                tc_fence_after();
                const uint64_t a = pd0 + (uint64_t)((j & 1) * kChunkUnits);
                const int vfirst = b * L::TILE_CHUNKS + (SEPV ? KC : 0);
#pragma unroll
                for (int gi = 0; gi < NG; ++gi) {
                    const int n = (NV - gi * 256) < 256 ? (NV - gi * 256) : 256;
                    umma_ss_k64_step(tmem + gi * 256, a, 2, vd0 + (uint64_t)((vfirst + gi * 4) * kChunkUnits), 128,
                                     idesc_bf16(SM_ROWS, n, false, true), j > 0);
                }
                umma_commit(&bars->kv_empty[b]);
                umma_commit(&bars->o_done);
            };
            // Out-of-order issue between two in-order streams: S(js) as soon as its tile
            // is gathered (and its TMEM buffer is free: S may run at most one tile ahead
            // of P V, the softmax of tile js-2 being done once P(js-2) was posted), else
            // O += P(jp) V(jp) as soon as P(jp) is posted.  The softmax of tile j then
            // runs under S(j+1) instead of leaving the tensor pipe idle, while P V never
            // waits behind a gather it does not need.  Bounded: no progress for
            // kWaitLimitNs ends the loop with an error.
            int js = 0, jp = 0;
            uint64_t t_last = globaltimer_ns();
            while (ok && jp < nt) {
                if (js < nt && js <= jp + 1 && mbar_test(&bars->kv_full[js % NSTG], (uint32_t)((js / NSTG) & 1))) {
                    issue_s(js++);
                    t_last = globaltimer_ns();
                } else if (jp < js && mbar_test(&bars->p_full[jp & 1], (uint32_t)((jp >> 1) & 1))) {
                    issue_pv(jp++);
                    t_last = globaltimer_ns();
                } else if (globaltimer_ns() - t_last > kWaitLimitNs) {
                    ok = false;
                }
            }
            if (!ok) report(p.status, ST_TIMEOUT_MMA);
            umma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0);
        }
    } else {
        // =============================== softmax and epilogue (warps 4-7)
        const int q4 = warp & 3;
        const int half = lane >> 4;             // which 32 of the 64 keys / columns
        const int r = q4 * 16 + (lane & 15);    // head row within the CTA
        const int h = h0 + r;
        const bool row_ok = h < p.H;
        const uint32_t o_lanes = (uint32_t)(q4 * 32) << 16;
        const float sl2 = p.scale_log2;
        float m_use = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            const int sb = j & 1, b = j % NSTG;
            ok = warp_all_sparse(mbar_wait(&bars->s_full[sb], (uint32_t)((j >> 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[32];
            tmem_ld16x2_32(tmem + o_lanes + TM_S + sb * SBN, sv);
            tmem_wait_ld();
            // validity of this thread's 32 keys, published with the tile (kv_full is
            // already complete here; waiting on it orders the mask read after its write)
            ok = warp_all_sparse(mbar_wait(&bars->kv_full[b], (uint32_t)((j / NSTG) & 1)));
            if (!ok) break;
            const uint32_t bits = bars->mask[b][half];
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (!((bits >> i) & 1u)) sv[i] = __float_as_uint(-INFINITY);
                mx = fmaxf(mx, __uint_as_float(sv[i]));
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16)) * sl2;
            const bool need = mx > m_use + S_RESCALE;
            float alpha = 1.f;
            if (need) {
                alpha = (m_use == -INFINITY) ? 0.f : fast_exp2(m_use - mx);
                m_use = mx;
            }
            const float msafe = (m_use == -INFINITY) ? 0.f : m_use;
            float rowsum = 0.f;
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * i]), sl2, -msafe));
                const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * i + 1]), sl2, -msafe));
                rowsum += p0 + p1;
                pk[i] = pack_bf16(p0, p1);
            }
            l = l * alpha + rowsum;   // this thread's half of the row; halves are added at the end
            // P row r, keys half*32 .. +31 = 16-byte units half*4 .. half*4+3 of P buffer
            // sb.  P V of tile j-2, the last reader of this buffer, completed before the
            // o_done wait of tile j-1.
            uint8_t *prow = sP + sb * L::P_BYTES;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                *reinterpret_cast<uint4 *>(prow + swz(r, half * 4 + u)) =
                    make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            fence_proxy_async_smem();
            if (j > 0) {
                ok = warp_all_sparse(mbar_wait(&bars->o_done, (uint32_t)((j - 1) & 1)));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                    for (int c = 0; c < VC; ++c) {
                        uint32_t ov[32];
                        tmem_ld16x2_32(tmem + o_lanes + c * 64, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st16x2_32(tmem + o_lanes + c * 64, ov);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[sb]);
        }
        if (ok && nt > 0) {
            ok = warp_all_sparse(mbar_wait(&bars->o_done, (uint32_t)((nt - 1) & 1)));
            tc_fence_after();
        }
        if (!ok) report(p.status, ST_TIMEOUT_SOFTMAX);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        float fac, lse;
        if (p.sinks && !p.part_o) {   // a split's partial leaves the sink to the merge
            const float sg = row_ok ? p.sinks[h] * S_LOG2E : 0.f;
            const float mf = fmaxf(m_use, sg);
            const float a = (m_use == -INFINITY) ? 0.f : exp2f(m_use - mf);
            const float lf = l * a + exp2f(sg - mf);
            fac = a / lf;
            lse = (mf + log2f(lf)) * S_LN2;
        } else {
            fac = l > 0.f ? 1.f / l : 0.f;
            lse = l > 0.f ? (m_use + log2f(l)) * S_LN2 : -INFINITY;
        }
        __nv_bfloat16 *orow = p.o + (int64_t)tok * p.os[0] + (int64_t)h * p.os[1];
        const int64_t prow = ((int64_t)sp * p.Sq + tok) * p.H + h;   // partial row (split calls)
#pragma unroll 1
        for (int c = 0; c < VC; ++c) {
            uint32_t ov[32];
            if (nt > 0 && ok) {
                tmem_ld16x2_32(tmem + o_lanes + c * 64, ov);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = 0u;
            }
            if (row_ok && p.part_o) {
                float4 *dst = reinterpret_cast<float4 *>(p.part_o + prow * p.Dv + c * 64 + half * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(__uint_as_float(ov[4 * i]) * fac, __uint_as_float(ov[4 * i + 1]) * fac,
                                         __uint_as_float(ov[4 * i + 2]) * fac, __uint_as_float(ov[4 * i + 3]) * fac);
            } else if (row_ok) {
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16(__uint_as_float(ov[2 * i]) * fac, __uint_as_float(ov[2 * i + 1]) * fac);
                uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 64 + half * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
        if (row_ok && half == 0) {
            if (p.part_o)
                p.part_lse[prow] = lse;
            else
                p.lse[(int64_t)tok * p.H + h] = lse;
        }
    }

    // Each warp arrives whole (a role branch may have left lanes behind, e.g. the MMA
    // issuer's lane 0), so the barrier below holds until every warp is done with TMEM.
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int KC, int VC, bool SEPV>
cudaError_t launch_sp(const SparseTcParams &p, cudaStream_t s)
{
    using L = SparseLayout<KC, VC, SEPV>;
    auto kern = sparse_tc_kernel<KC, VC, SEPV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    if (p.splits < 1 || (p.splits > 1 && (!p.part_o || !p.part_lse)) || p.chunk < 1) return cudaErrorInvalidValue;
    const int grid = p.Sq * ((p.H + SM_ROWS - 1) / SM_ROWS) * p.splits;
    kern<<<grid, S_THREADS, L::BYTES, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

int sparse_smem_bytes(int dqk, int dv, bool sepv)
{
    const int kc = dqk / 64, vc = dv / 64;
    const int tile = (kc + (sepv ? vc : 0)) * SCHUNK;
    return 1024 + NSTG * tile + 2 * SCHUNK + (int)sizeof(SparseBars);
}

bool sparse_tc_supported(int dqk, int dv, bool sepv)
{
#define ARC_SP(K, V, S) if (dqk == K * 64 && dv == V * 64 && sepv == S) return true;
    ARC_SP(8, 8, false) ARC_SP(8, 4, false) ARC_SP(4, 4, false) ARC_SP(2, 2, false) ARC_SP(2, 1, true)
    ARC_SP(2, 2, true) ARC_SP(4, 4, true)
#undef ARC_SP
    return false;
}

cudaError_t launch_sparse_tc(const SparseTcParams &p, cudaStream_t s)
{
    const bool sepv = p.v != nullptr;
#define ARC_SP(K, V, S) \
    if (p.Dqk == K * 64 && p.Dv == V * 64 && sepv == S) return launch_sp<K, V, S>(p, s);
    ARC_SP(8, 8, false) ARC_SP(8, 4, false) ARC_SP(4, 4, false) ARC_SP(2, 2, false) ARC_SP(2, 1, true)
    ARC_SP(2, 2, true) ARC_SP(4, 4, true)
#undef ARC_SP
    return cudaErrorInvalidValue;
}

}  // namespace arc
