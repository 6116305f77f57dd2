// attn_pair.cu -- attention forward on a pair of CTAs (cta_group::2), for
// head dims where one CTA's shared memory is mostly taken by its Q tile
// (d_qk = 512: 128 query rows x 512 = 128 KB), for d_qk 128-256 with d_v 128,
// and for MLA prefill
// (d_qk 128 + 64, d_v 128: one d_v pass, Q and K concatenated on load from
// the nope and the shared rope tensors).  With M = 256 each CTA reads only half
// of every B operand from its shared memory, which keeps the S = Q K^T MMAs of
// the small head dims below the shared-memory bandwidth (an M = 128, N = 128
// SS MMA reads 8 KB per 64 clk, all of it).
//
// A cluster of two CTAs owns 256 consecutive fold rows of one (batch, kv head)
// group and one d_v slice; each CTA keeps its own 128 rows of Q and of O.  The
// leader CTA (rank 0) issues every MMA for the pair with M = 256:
//   S = Q K^T   N = 128 keys: each CTA stages 64 of the tile's keys
//   O += P V    N = 128 d_v columns per MMA: each CTA stages 64 of them,
//               P is each CTA's own TMEM (the A operand of its rows)
// so every K/V byte a CTA brings from L2 feeds 256 query rows: half the
// per-SM load traffic of the single-CTA kernel for the same tensor work.
//
// Synchronisation across the pair
//   - both CTAs' TMA loads signal the leader's `full` barrier (2-SM form of the
//     bulk tensor copy); the leader's producer posts the expected bytes of both
//   - the leader's tcgen05.commit arrives on the barrier at the same offset in
//     both CTAs (empty stages, S ready, O done)
//   - every softmax thread of both CTAs arrives on the leader's `p_full`
//   - cluster barriers after set-up and before TMEM is released
// Loads are plain (no multicast); only the commit arrive is multicast.
// Every mbarrier wait is bounded and reports through p.status.
#include <math.h>

#include <algorithm>

#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace arc {
namespace {

constexpr int PBM = 128;           // query rows per CTA
constexpr int PBN = 128;           // keys per KV tile (64 staged by each CTA)
constexpr int PCH = 64 * 128;      // bytes of one [64 rows x 64 bf16] swizzled box
constexpr int BPS = 4;             // boxes per ring stage (one barrier hand-off per 32 KB)
constexpr int PST = BPS * PCH;     // bytes of one ring stage
constexpr int P_THREADS = 256;
constexpr int P_TMEM = 512;
constexpr int P_SCOL = 256;        // S/P double buffer at columns 256, 384
constexpr int P_MAX_STAGES = 16;
constexpr int P_SMEM_LIMIT = 232448;
constexpr float P_LOG2E = 1.4426950408889634f;
constexpr float P_LN2 = 0.6931471805599453f;
constexpr float P_RESCALE = 8.0f;

struct PairBars {
    uint64_t q_full;
    uint64_t q_empty;   // the last S of a row tile has read Q: the next tile's Q may land
    uint64_t s_full[2];
    uint64_t p_full;
    uint64_t o_done;
    uint64_t drain;
    uint64_t full[P_MAX_STAGES];
    uint64_t empty[P_MAX_STAGES];
    uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on the leader's barrier from the other CTA of the pair.  The data this
// orders is in TMEM and is ordered by the tcgen05 fences around the arrive and
// the wait; a release at cluster scope (which costs ~1-2k clk here) is not needed.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 2-SM bulk tensor loads: data lands in this CTA's shared memory, the
// transaction bytes are counted on the barrier at `mbar_cluster` (the leader's).
__device__ __forceinline__ void tma2_load_3d(void *dst, const CUtensorMap *map, uint32_t mbar_cluster, int c0, int c1,
                                             int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(mbar_cluster), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma2_load_4d(void *dst, const CUtensorMap *map, uint32_t mbar_cluster, int c0, int c1,
                                             int c2, int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(mbar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tma2_load_5d(void *dst, const CUtensorMap *map, uint32_t mbar_cluster, int c0, int c1,
                                             int c2, int c3, int c4)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(mbar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx_u32(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// Commit of the pair's MMAs: arrive once on the barrier at this offset in both CTAs.
__device__ __forceinline__ void umma2_commit_both(uint64_t *bar)
{
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void umma2_ss_k64(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 q, %4, %4;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %5, %6, %3, q;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %7, %8, %3, q;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %9, %10, %3, q;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "l"(a + 2), "l"(b + 2), "l"(a + 4), "l"(b + 4), "l"(a + 6), "l"(b + 6)
        : "memory");
}

__device__ __forceinline__ void umma2_ts_k64(uint32_t d, uint32_t a_tm, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 q, %4, %4;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%5], %6, %3, q;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%7], %8, %3, q;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%9], %10, %3, q;\n\t}" ::"r"(d),
        "r"(a_tm), "l"(b), "r"(idesc), "r"(acc), "r"(a_tm + 8), "l"(b + 128), "r"(a_tm + 16), "l"(b + 256),
        "r"(a_tm + 24), "l"(b + 384)
        : "memory");
}

// Wait on a barrier of this CTA whose arrivals were released at cluster scope
// by the other CTA of the pair (p_full).  Bounded like mbar_wait.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

__device__ __forceinline__ bool warp_all_pair(bool ok) { return __all_sync(0xffffffffu, ok); }

// The k-th item of cluster c out of C: items are ordered by decreasing work, and
// round k hands them out left to right on even rounds and right to left on odd
// ones, which evens out the clusters' totals.  Increases with k for every c.
__device__ __forceinline__ int snake_item(int k, int c, int C) { return k * C + ((k & 1) ? C - 1 - c : c); }

// One work item of the persistent pair kernel: 256 consecutive fold rows (rp ..)
// of kv head kv of batch b, and the number of 128-key tiles they need.
struct PairItem {
    int b, kv, rp, nt;
};

__device__ __forceinline__ PairItem pair_item(const TcParams &p, int item)
{
    const int groups = p.B * p.Hkv;
    const int prank = item / groups, rest = item % groups;
    PairItem w;
    w.kv = rest % p.Hkv;
    w.b = rest / p.Hkv;
    const int pair = prank < 1024 ? (int)p.tile_order[prank] : prank;
    const int rows_in_group = p.G * p.Tq;
    w.rp = pair * 2 * PBM;
    const int r_last = min(w.rp + 2 * PBM, rows_in_group) - 1;
    const int t_max = p.tmajor ? r_last / p.G : ((w.rp / p.Tq != r_last / p.Tq) ? p.Tq - 1 : r_last % p.Tq);
    const int kv_last = p.causal ? min(p.Tk - 1, t_max + p.Tk - p.Tq) : p.Tk - 1;
    w.nt = kv_last < 0 ? 0 : kv_last / PBN + 1;
    return w;
}

// One 32-byte global store (a whole sector); dst must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void *dst, const uint32_t *w)
{
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                 "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

template <int DQK, int DVS, bool MLA>
__global__ void __launch_bounds__(P_THREADS, 1) tc_attn_pair_kernel(const __grid_constant__ TcParams p)
{
    constexpr int KC = DQK / 64;     // 64-column chunks of a Q / K row
    constexpr int VG = DVS / 128;    // 128-column MMA groups of the d_v slice
    // Boxes per ring stage: BPS when a tile's boxes are a multiple of it, else the
    // whole tile in one partly filled stage (d_qk 192: 3 K boxes; d_v 128: 2 V boxes).
    constexpr int KB = (KC % BPS == 0) ? BPS : KC;
    constexpr int VB = ((2 * VG) % BPS == 0) ? BPS : 2 * VG;
    static_assert(DQK % 64 == 0 && DVS % 128 == 0 && DVS <= 256, "tile shape");
    static_assert(KB <= BPS && KC % KB == 0 && VB <= BPS && (2 * VG) % VB == 0, "K and V tiles fill ring stages");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem<1024>(smem_raw);
    uint8_t *sQ = smem;                          // KC chunks of [128 rows x 64]
    uint8_t *sRing = sQ + KC * 2 * PCH;          // R stages of BPS boxes of [64 rows x 64]
    const int R = p.stages;
    PairBars *bars = reinterpret_cast<PairBars *>(sRing + R * PST);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;

    // ---- persistent schedule: cluster c takes one item per round of a list ordered by
    // decreasing work (snake order, see snake_item).  Within an item the pair computes every d_v slice
    // of its rows in turn with Q resident: unit u of the item is (slice u / nt, key
    // tile u % nt); units are numbered globally across items (S buffer u & 1 and
    // the barrier parities follow the global number).
    const int C = gridDim.x >> 1, c0 = blockIdx.x >> 1;
    const int n_items = ((p.n_tiles + 1) / 2) * p.B * p.Hkv;
    const int NSL = p.n_slices;
    const int rows_in_group = p.G * p.Tq;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int i = 0; i < 2; ++i) mbar_init(&bars->s_full[i], 1);
        mbar_init(&bars->p_full, 256);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        for (int i = 0; i < R; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], 1);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&bars->tmem_base)),
                     "r"(P_TMEM)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // =============================== TMA producer (both CTAs, each its half)
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_q);
            tma_prefetch_desc(&p.tm_k);
            tma_prefetch_desc(&p.tm_v);
            const uint32_t q_full_l = mapa(smem_u32(&bars->q_full), 0);
            int stage = 0, qn = 0;
            uint32_t ephase = 0;
            bool ok = true;
            // Each barrier round trip costs this thread a few hundred clocks, so a
            // stage carries BPS boxes: one wait and one expect_tx per 32 KB.
            auto acquire = [&](int boxes) -> bool {
                if (!mbar_wait(&bars->empty[stage], ephase ^ 1u)) return false;
                if (leader) mbar_arrive_expect_tx_u32(smem_u32(&bars->full[stage]), 2 * boxes * PCH);
                return true;
            };
            auto advance = [&]() {
                if (++stage == R) {
                    stage = 0;
                    ephase ^= 1u;
                }
            };
            auto full_l = [&]() { return mapa(smem_u32(&bars->full[stage]), 0); };
            for (int k = 0; ok && snake_item(k, c0, C) < n_items; ++k) {
                const PairItem w = pair_item(p, snake_item(k, c0, C));
                if (w.nt == 0) continue;
                const int nt = w.nt, NI = nt * NSL, kv = w.kv, b = w.b;
                const int r0 = w.rp + (int)rank * PBM;
                // Q of this item replaces the previous item's once its last S has run
                if (qn > 0 && !(ok = mbar_wait(&bars->q_empty, (uint32_t)((qn - 1) & 1)))) break;
                if (leader) mbar_arrive_expect_tx_u32(smem_u32(&bars->q_full), 2 * KC * 2 * PCH);
                if (p.tmajor) {
                    // box {64, G, 128/G}: smem row = (t - t0) * G + head in group
                    for (int c = 0; c < KC; ++c)
                        tma2_load_5d(sQ + c * 2 * PCH, &p.tm_q, q_full_l, c * 64, 0, r0 / p.G, kv, b);
                } else {
                    const int qrow = kv * rows_in_group + r0;
                    for (int c = 0; c < KC; ++c) {
                        if (!MLA || c < p.kc_first)
                            tma2_load_3d(sQ + c * 2 * PCH, &p.tm_q, q_full_l, c * 64, qrow, b);
                        else   // MLA: the rope columns of q
                            tma2_load_3d(sQ + c * 2 * PCH, &p.tm_q2, q_full_l, (c - p.kc_first) * 64, qrow, b);
                    }
                }
                ++qn;
                auto load_k = [&](int j) -> bool {
                    for (int cc = 0; cc < KC; cc += KB) {
                        if (!acquire(KB)) return false;
                        const uint32_t fl = full_l();
                        for (int q = 0; q < KB; ++q) {
                            const int c = cc + q;
                            if (!MLA || c < p.kc_first)
                                tma2_load_4d(sRing + stage * PST + q * PCH, &p.tm_k, fl, c * 64,
                                             j * PBN + (int)rank * 64, kv, b);
                            else   // MLA: the rope columns, shared by every head
                                tma2_load_3d(sRing + stage * PST + q * PCH, &p.tm_k2, fl, (c - p.kc_first) * 64,
                                             j * PBN + (int)rank * 64, b);
                        }
                        advance();
                    }
                    return true;
                };
                // V box q of a stage: 128-column group q / 2, key half q % 2
                auto load_v = [&](int it) -> bool {
                    const int j = it % nt, dv0 = (it / nt) * DVS;
                    for (int q0 = 0; q0 < 2 * VG; q0 += VB) {
                        if (!acquire(VB)) return false;
                        const uint32_t fl = full_l();
                        for (int q = 0; q < VB; ++q) {
                            const int g = (q0 + q) >> 1, hh = (q0 + q) & 1;
                            tma2_load_4d(sRing + stage * PST + q * PCH, &p.tm_v, fl, dv0 + g * 128 + (int)rank * 64,
                                         j * PBN + hh * 64, kv, b);
                        }
                        advance();
                    }
                    return true;
                };
                ok = load_k(0);
                for (int it = 0; ok && it < NI; ++it) {
                    if (it + 1 < NI) ok = load_k((it + 1) % nt);
                    if (ok) ok = load_v(it);
                }
            }
            if (!ok) report(p.status, ST_TIMEOUT_LOAD);
        }
    } else if (warp == 1) {
        // =============================== MMA issuer (leader only)
        if (leader && lane == 0) {
            constexpr uint32_t kBox = PCH >> 4;       // descriptor units per 8 KB box
            const uint32_t idesc_s = idesc_bf16(2 * PBM, PBN, false, false);
            const uint32_t idesc_pv = idesc_bf16(2 * PBM, 128, false, true);
            const uint64_t qd0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t kd0 = sdesc_sw128(smem_u32(sRing), 16, 1024);
            const uint64_t vd0 = sdesc_sw128(smem_u32(sRing), 16, 1024);
            int stage = 0, qn = 0, gu = 0;
            uint32_t fphase = 0;
            bool ok = true;
            auto advance = [&]() {
                if (++stage == R) {
                    stage = 0;
                    fphase ^= 1u;
                }
            };
            // A shared-memory access by this thread after a tcgen05.commit waits
            // until the committed MMAs have completed, so every barrier wait here
            // empties the tensor pipe (measured: ~230 clk of idle pipe per wait).
            // The issuer therefore waits once for a whole operand tile (all K
            // boxes of S, or P plus all V boxes of PV) and then issues the tile's
            // MMAs back to back; ring boxes are still released one by one.
            auto wait_boxes = [&](int n) -> bool {
                int st = stage;
                uint32_t ph = fphase;
                for (int i = 0; i < n; ++i) {
                    if (!mbar_wait(&bars->full[st], ph)) return false;
                    if (++st == R) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
                return true;
            };
            auto issue_s = [&](int it) -> bool {
                const uint32_t d = tmem + P_SCOL + (it & 1) * PBN;
                if (!wait_boxes(KC / KB)) return false;
                tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < KC; c0 += KB) {
#pragma unroll
                    for (int q = 0; q < KB; ++q)
                        umma2_ss_k64(d, qd0 + (uint64_t)((c0 + q) * 2 * kBox), kd0 + (uint64_t)((stage * BPS + q) * kBox),
                                     idesc_s, (c0 + q) > 0);
                    umma2_commit_both(&bars->empty[stage]);
                    advance();
                }
                umma2_commit_both(&bars->s_full[it & 1]);
                return true;
            };
            auto issue_pv = [&](int it, bool first) -> bool {   // first key tile of a slice overwrites O
                if (!mbar_wait_cluster(&bars->p_full, (uint32_t)(it & 1))) return false;
                if (!wait_boxes(2 * VG / VB)) return false;
                tc_fence_after();
                const uint32_t p_tm = tmem + P_SCOL + (it & 1) * PBN;
#pragma unroll 1
                for (int q0 = 0; q0 < 2 * VG; q0 += VB) {
#pragma unroll
                    for (int q = 0; q < VB; ++q) {
                        const int g = (q0 + q) >> 1, hh = (q0 + q) & 1;
                        umma2_ts_k64(tmem + g * 128, p_tm + hh * 32, vd0 + (uint64_t)((stage * BPS + q) * kBox), idesc_pv,
                                     (first ? 0 : 1) | hh);
                    }
                    umma2_commit_both(&bars->empty[stage]);
                    advance();
                }
                umma2_commit_both(&bars->o_done);
                return true;
            };
            for (int k = 0; ok && snake_item(k, c0, C) < n_items; ++k) {
                const PairItem w = pair_item(p, snake_item(k, c0, C));
                if (w.nt == 0) continue;
                const int nt = w.nt, NI = nt * NSL;
                if (!(ok = mbar_wait(&bars->q_full, (uint32_t)(qn & 1)))) break;
                tc_fence_after();
                ++qn;
                // units gu .. gu + NI - 1; the last S of the item frees Q for the next one
                ok = issue_s(gu);
                if (ok && NI == 1) umma2_commit_both(&bars->q_empty);
                for (int it = 0; ok && it < NI; ++it) {
                    if (it + 1 < NI) {
                        ok = issue_s(gu + it + 1);
                        if (ok && it + 2 == NI) umma2_commit_both(&bars->q_empty);
                    }
                    if (ok) ok = issue_pv(gu + it, (it % nt) == 0);
                }
                gu += NI;
            }
            if (!ok) report(p.status, ST_TIMEOUT_MMA);
            umma2_commit_both(&bars->drain);
        }
    } else if (warp >= 4) {
        // =============================== softmax and epilogue (both CTAs, own rows)
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const float sl2 = p.scale_log2;
        const uint32_t p_full_l = mapa(smem_u32(&bars->p_full), 0);
        bool ok = true;
        int gu = 0;
        for (int k = 0; ok && snake_item(k, c0, C) < n_items; ++k) {
        const PairItem w = pair_item(p, snake_item(k, c0, C));
        const int nt = w.nt, kv = w.kv, b = w.b;
        const int R_ = w.rp + (int)rank * PBM + r;
        const bool row_ok = R_ < rows_in_group;
        const int t = p.tmajor ? R_ / p.G : R_ % p.Tq;
        const int h = kv * p.G + (p.tmajor ? R_ % p.G : R_ / p.Tq);
        const int last = p.causal ? min(p.Tk - 1, t + p.Tk - p.Tq) : p.Tk - 1;
        // The row max and sum come from the first d_v slice; later slices recompute
        // the same S and reuse them: with the lazy max fixed, p = exp2(s - m_use) <= 2^8,
        // so no running max, row sum or O rescale is needed there.
        float m_use = -INFINITY, l = 0.f;
        for (int slice = 0; ok && slice < NSL; ++slice) {
        const int dv0 = slice * DVS;
        const bool first = slice == 0;
        for (int j = 0; ok && j < nt; ++j) {
            const int it = gu + slice * nt + j;
            const int buf = it & 1;
            const uint32_t s_tmem = tmem + lane_off + P_SCOL + buf * PBN;
            ok = warp_all_pair(mbar_wait(&bars->s_full[buf], (uint32_t)((it >> 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[PBN];
#pragma unroll
            for (int i = 0; i < PBN / 32; ++i)
                tmem_ld32(s_tmem + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * i]));
            tmem_wait_ld();
            const int kbase = j * PBN;
            if (kbase + PBN - 1 > last) {
#pragma unroll
                for (int i = 0; i < PBN; ++i)
                    if (kbase + i > last) sv[i] = __float_as_uint(-INFINITY);
            }
            float alpha = 1.f;
            if (first) {
                float mx = -INFINITY;
#pragma unroll
                for (int i = 0; i < PBN; ++i) mx = fmaxf(mx, __uint_as_float(sv[i]));
                mx *= sl2;
                if (mx > m_use + P_RESCALE) {
                    alpha = (m_use == -INFINITY) ? 0.f : fast_exp2(m_use - mx);
                    m_use = mx;
                }
            }
            const float msafe = (m_use == -INFINITY) ? 0.f : m_use;
            // P = exp2(S*scale - m) as bf16 over S in place; the row sum only in the first slice
            auto p_tile = [&](auto with_sum) {
                float rowsum = 0.f;
#pragma unroll
                for (int c = 0; c < PBN / 8; ++c) {
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float p0 = fast_exp2(fmaf(__uint_as_float(sv[8 * c + 2 * i]), sl2, -msafe));
                        const float p1 = fast_exp2(fmaf(__uint_as_float(sv[8 * c + 2 * i + 1]), sl2, -msafe));
                        if constexpr (decltype(with_sum)::value) rowsum += p0 + p1;
                        pk[i] = pack_bf16(p0, p1);
                    }
                    tmem_st4(s_tmem + 4 * c, pk[0], pk[1], pk[2], pk[3]);
                }
                return rowsum;
            };
            if (first)
                l = l * alpha + p_tile(std::true_type{});
            else
                p_tile(std::false_type{});
            if (j > 0) {
                ok = warp_all_pair(mbar_wait(&bars->o_done, (uint32_t)((it - 1) & 1)));
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
            if (leader)
                mbar_arrive(&bars->p_full);
            else
                mbar_arrive_remote(p_full_l);
        }
        if (ok && nt > 0) {
            ok = warp_all_pair(mbar_wait(&bars->o_done, (uint32_t)((gu + slice * nt + nt - 1) & 1)));
            tc_fence_after();
        }
        float fac, lse;
        if (p.sinks) {
            const float sg = row_ok ? p.sinks[h] * P_LOG2E : 0.f;
            const float mf = fmaxf(m_use, sg);
            const float a = (m_use == -INFINITY) ? 0.f : exp2f(m_use - mf);
            const float lf = l * a + exp2f(sg - mf);
            fac = a / lf;
            lse = (mf + log2f(lf)) * P_LN2;
        } else {
            fac = l > 0.f ? 1.f / l : 0.f;
            lse = l > 0.f ? (m_use + log2f(l)) * P_LN2 : -INFINITY;
        }
        __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(p.o) + (int64_t)b * p.os[0] + (int64_t)h * p.os[1] +
                              (int64_t)t * p.os[2] + dv0;
        // Four 32-column TMEM loads in flight per wait; each 32-column piece of
        // the row leaves as two 32-byte stores (whole sectors).
        const bool st32 = (reinterpret_cast<uintptr_t>(orow) & 31) == 0;
#pragma unroll 1
        for (int c0 = 0; c0 < DVS / 32; c0 += 4) {
            uint32_t ov[4][32];
            if (nt > 0 && ok) {
#pragma unroll
                for (int u = 0; u < 4; ++u) tmem_ld32(tmem + lane_off + 32 * (c0 + u), ov[u]);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[u][i] = 0u;
            }
            if (row_ok) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[i] = pack_bf16(__uint_as_float(ov[u][2 * i]) * fac, __uint_as_float(ov[u][2 * i + 1]) * fac);
                    __nv_bfloat16 *dst = orow + 32 * (c0 + u);
                    if (st32) {
                        st_global_v8(dst, w);
                        st_global_v8(dst + 16, w + 8);
                    } else {
                        uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                    }
                }
            }
        }
        if (row_ok && slice == 0) p.lse[((int64_t)b * p.H + h) * p.Tq + t] = lse;
        }
        gu += nt * NSL;
        }
        if (!ok) report(p.status, ST_TIMEOUT_SOFTMAX);
    }

    // Drain: the leader's last MMAs have finished (they write both CTAs' TMEM)
    // and their final commit has reached this CTA's barriers before either CTA
    // leaves; then release TMEM.
    __syncwarp();
    if (warp == 1 && lane == 0) mbar_wait(&bars->drain, 0);
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(P_TMEM) : "memory");
    }
    cluster_sync_all();
}

template <int DQK, int DVS, bool MLA>
cudaError_t launch_p(const TcParams &p, int grid, cudaStream_t s)
{
    const int smem = pair_smem_bytes(DQK, p.stages);
    auto kern = tc_attn_pair_kernel<DQK, DVS, MLA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(P_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Persistent: as many clusters as can be resident at once (each walks the item list).
    cfg.gridDim = dim3(2);
    int resident = 0;
    if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess || resident <= 0) {
        cudaGetLastError();
        resident = grid / 2;
    }
    const int clusters = std::max(1, std::min(grid / 2, resident));
    cfg.gridDim = dim3(2 * clusters);
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

int pair_smem_bytes(int dqk, int stages) { return 1024 + (dqk / 64) * 2 * PCH + stages * PST + (int)sizeof(PairBars); }

int pair_max_stages(int dqk)
{
    int st = (P_SMEM_LIMIT - 1024 - (int)sizeof(PairBars) - (dqk / 64) * 2 * PCH) / PST;
    return st < P_MAX_STAGES ? st : P_MAX_STAGES;
}

bool pair_supported(int dqk, int dvs, bool mla)
{
    if (mla) return dqk == 192 && dvs == 128;
    return ((dqk == 512 || dqk == 256) && dvs == 256) || ((dqk == 128 || dqk == 192 || dqk == 256) && dvs == 128);
}

cudaError_t launch_tc_attn_pair(const TcParams &p, int dqk, int dvs, bool mla, int grid, cudaStream_t s)
{
    if (!mla && dqk == 512 && dvs == 256) return launch_p<512, 256, false>(p, grid, s);
    if (!mla && dqk == 256 && dvs == 256) return launch_p<256, 256, false>(p, grid, s);
    if (!mla && dqk == 256 && dvs == 128) return launch_p<256, 128, false>(p, grid, s);
    if (!mla && dqk == 192 && dvs == 128) return launch_p<192, 128, false>(p, grid, s);
    if (!mla && dqk == 128 && dvs == 128) return launch_p<128, 128, false>(p, grid, s);
    if (mla && dqk == 192 && dvs == 128) return launch_p<192, 128, true>(p, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace arc
