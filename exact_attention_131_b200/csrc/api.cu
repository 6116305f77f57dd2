// api.cu -- the C ABI declared in include/arc_attn.h: host-side validation,
// planning (which kernel, which tiling), TMA descriptor encoding and launch.
// Nothing here allocates device memory; nothing is launched when validation
// fails.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

using namespace arc;

namespace {

constexpr int kTcBM = 128, kTcBN = 128;
constexpr float kLog2e = 1.4426950408889634f;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A zero stride over an extent above one: a broadcast view of an input (legal for the
// CUDA-core kernels, which index it as given; a TMA tensor map cannot describe it), or
// output rows that would alias one another (refused everywhere).
bool broadcast(int64_t stride, int64_t extent) { return stride == 0 && extent > 1; }
bool in_set(int x, std::initializer_list<int> s) { return std::find(s.begin(), s.end(), x) != s.end(); }

// The softmax scale a call computes with: 1/sqrt(d_qk) under ARC_FLAG_DEFAULT_SCALE
// (evaluated in double, then rounded once to fp32), otherwise the caller's value.
float call_scale(uint32_t flags, float scale, int dqk)
{
    return (flags & ARC_FLAG_DEFAULT_SCALE) ? (float)(1.0 / sqrt((double)dqk)) : scale;
}

// A NaN scale is refused unless the flag replaces it.
bool scale_ok(uint32_t flags, float scale) { return (flags & ARC_FLAG_DEFAULT_SCALE) || scale == scale; }

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

void set_name(arc_plan_info *pi, const char *name)
{
    memset(pi, 0, sizeof(*pi));
    snprintf(pi->kernel, sizeof(pi->kernel), "%s", name);
}

bool log_enabled()
{
    const char *e = getenv("ARC_LOG");
    return e && e[0] == '1';
}

// First dispatch per kernel name is logged when ARC_LOG=1 (host-side logging
// only; it never influences what a call computes).
void note_dispatch(const char *kernel)
{
    if (!log_enabled()) return;
    static std::mutex mu;
    static std::vector<std::string> seen;
    std::lock_guard<std::mutex> lock(mu);
    for (auto &s : seen)
        if (s == kernel) return;
    seen.emplace_back(kernel);
    fprintf(stderr, "arc_attn: first dispatch on %s\n", kernel);
}

// ------------------------------------------------------------------ TMA maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// bf16 tensor map, 128-byte swizzle, box {64, rows, 1...}; dims/strides innermost first,
// strides in elements for dims 1..rank-1.
bool make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims, const int64_t *strides_el,
              uint32_t box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[5], gstr[4];
    cuuint32_t box[5], estr[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        estr[i] = 1;
        box[i] = i == 0 ? 64 : (i == 1 ? box_rows : 1);
    }
    for (int i = 0; i < rank - 1; ++i) gstr[i] = (cuuint64_t)strides_el[i] * 2;
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), gdim, gstr, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Same with an explicit box (one entry per dimension, innermost first).
bool make_map_box(CUtensorMap *m, const void *base, int rank, const uint64_t *dims, const int64_t *strides_el,
                  const uint32_t *box_in)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[5], gstr[4];
    cuuint32_t box[5], estr[5];
    for (int i = 0; i < rank; ++i) gdim[i] = dims[i], estr[i] = 1, box[i] = box_in[i];
    for (int i = 0; i < rank - 1; ++i) gstr[i] = (cuuint64_t)strides_el[i] * 2;
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), gdim, gstr, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Byte tensor {width bytes, rows}, row stride = width, no swizzle; box {box_w bytes, box_rows}.
bool make_map_bytes(CUtensorMap *m, const void *base, uint64_t width, uint64_t rows, uint32_t box_w, uint32_t box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {width, rows}, gstr[1] = {width};
    cuuint32_t box[2] = {box_w, box_rows}, estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), gdim, gstr, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The decode caches are the same few buffers call after call, so their byte-tensor maps
// are kept: a map is a pure function of (base, width, rows, box), which is the key.
bool make_map_bytes_cached(CUtensorMap *m, const void *base, uint64_t width, uint64_t rows, uint32_t box_w,
                           uint32_t box_rows)
{
    struct Entry {
        const void *base;
        uint64_t width, rows;
        uint32_t box_w, box_rows;
        CUtensorMap map;
    };
    static std::mutex mu;
    static Entry cache[16];
    static int used = 0, next = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i) {
            const Entry &e = cache[i];
            if (e.base == base && e.width == width && e.rows == rows && e.box_w == box_w && e.box_rows == box_rows) {
                *m = e.map;
                return true;
            }
        }
    }
    if (!make_map_bytes(m, base, width, rows, box_w, box_rows)) return false;
    std::lock_guard<std::mutex> lock(mu);
    Entry &e = cache[next];
    e.base = base, e.width = width, e.rows = rows, e.box_w = box_w, e.box_rows = box_rows, e.map = *m;
    next = (next + 1) % 16;
    used = std::max(used, next == 0 ? 16 : next);
    return true;
}

bool tma_strides_ok(std::initializer_list<int64_t> strides_el)
{
    for (int64_t s : strides_el)
        if (s <= 0 || (s * 2) % 16 != 0 || s * 2 >= (int64_t(1) << 40)) return false;
    return true;
}

// Tile order: heavier tiles (more KV tiles under the causal mask) first.
void order_tiles(TcParams &p, int n_tiles, int rows_per_item = kTcBM)
{
    if (n_tiles > 1024) {
        for (int i = 0; i < 1024; ++i) p.tile_order[i] = (uint16_t)i;
        return;
    }
    std::vector<std::pair<int, int>> w(n_tiles);
    const int rows = p.G * p.Tq;
    for (int t = 0; t < n_tiles; ++t) {
        const int r0 = t * rows_per_item, r_last = std::min(r0 + rows_per_item, rows) - 1;
        const int t_max = p.tmajor ? r_last / p.G : ((r0 / p.Tq != r_last / p.Tq) ? p.Tq - 1 : r_last % p.Tq);
        const int last = p.causal ? std::min(p.Tk - 1, t_max + p.Tk - p.Tq) : p.Tk - 1;
        w[t] = {last < 0 ? 0 : last / kTcBN + 1, t};
    }
    std::stable_sort(w.begin(), w.end(), [](auto &a, auto &b) { return a.first > b.first; });
    for (int i = 0; i < n_tiles; ++i) p.tile_order[i] = (uint16_t)w[i].second;
    for (int i = n_tiles; i < 1024; ++i) p.tile_order[i] = (uint16_t)i;
}

// ------------------------------------------------------------------ dense

bool tc_pair_supported(int dqk, int dvs, bool mla)
{
    static const int dense[][2] = {{64, 64}, {128, 64}, {128, 128}, {192, 128}, {256, 128},
                                   {256, 256}, {512, 256}, {512, 128}};
    static const int mlas[][2] = {{128, 128}, {192, 128}, {192, 64}, {256, 128}, {256, 256}};
    if (mla) {
        for (auto &x : mlas)
            if (x[0] == dqk && x[1] == dvs) return true;
    } else {
        for (auto &x : dense)
            if (x[0] == dqk && x[1] == dvs) return true;
    }
    return false;
}

arc_status check_attn(const arc_attn_args *a)
{
    if (!a) return ARC_ERR_INVALID_ARG;
    if (a->dtype != ARC_DTYPE_BF16 && a->dtype != ARC_DTYPE_F32) return ARC_ERR_INVALID_ARG;
    if (a->B < 0 || a->H <= 0 || a->Hkv <= 0 || a->H % a->Hkv || a->Tq < 0 || a->Tk < 0) return ARC_ERR_INVALID_ARG;
    if (a->D <= 0 || a->Dv <= 0 || a->D > 512 || a->Dv > 512) return ARC_ERR_UNSUPPORTED;
    if (a->B == 0 || a->Tq == 0) return ARC_OK;
    if (!a->q || !a->o || !a->lse || (a->Tk > 0 && (!a->k || !a->v))) return ARC_ERR_INVALID_ARG;
    if (!scale_ok(a->flags, a->scale)) return ARC_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        if (a->q_strides[i] < 0 || a->k_strides[i] < 0 || a->v_strides[i] < 0 || a->o_strides[i] < 0)
            return ARC_ERR_INVALID_ARG;
    if (broadcast(a->o_strides[0], a->B) || broadcast(a->o_strides[1], a->H) || broadcast(a->o_strides[2], a->Tq))
        return ARC_ERR_INVALID_ARG;
    return ARC_OK;
}

enum class Path { None, Simple, Tc };

struct AttnPlan {
    Path path = Path::None;
    bool two = false;   // two query tiles per CTA (d_v <= 128)
    bool pair = false;  // CTA pair, M = 256 (see pair_supported)
    int dvs = 0, n_slices = 0, n_tiles = 0, grid = 0, stages = 0;
};

bool tc2_pair_supported(int dqk, int dvs, bool mla)
{
    static const int dense[][2] = {{64, 64}, {128, 64}, {128, 128}, {192, 128}, {256, 128}};
    static const int mlas[][2] = {{128, 128}, {192, 128}, {192, 64}, {256, 128}};
    if (mla) {
        for (auto &x : mlas)
            if (x[0] == dqk && x[1] == dvs) return true;
    } else {
        for (auto &x : dense)
            if (x[0] == dqk && x[1] == dvs) return true;
    }
    return false;
}

// Switch a planned one-tile launch to the two-tile kernel when it applies.
void maybe_two(AttnPlan &pl, int dqk, bool mla, int groups)
{
    if (pl.dvs > 128 || pl.n_slices != 1 || !tc2_pair_supported(dqk, pl.dvs, mla)) return;
    const int st = tc2_max_stages(dqk);
    if (st < dqk / 64 + pl.dvs / 64) return;
    pl.two = true;
    pl.stages = st;
    pl.grid = ((pl.n_tiles + 1) / 2) * groups;
}

AttnPlan plan_attn(const arc_attn_args *a)
{
    AttnPlan pl;
    if (a->B == 0 || a->Tq == 0) return pl;
    const bool force_simple = (a->flags & ARC_FLAG_FORCE_SIMPLE) != 0;
    if (a->dtype == ARC_DTYPE_F32 || force_simple || a->Tk == 0) {
        if (a->D <= 512 && a->Dv <= 512) pl.path = Path::Simple;
        return pl;
    }
    pl.dvs = a->Dv > 256 ? 256 : a->Dv;
    pl.n_slices = (a->Dv + pl.dvs - 1) / pl.dvs;
    if (a->Dv % pl.dvs || !tc_pair_supported(a->D, pl.dvs, false)) return pl;
    // the fold view needs the g*Tq rows of a kv group evenly spaced
    if (a->q_strides[1] != (int64_t)a->Tq * a->q_strides[2] && a->H > 1) return pl;
    if (broadcast(a->q_strides[0], a->B) || broadcast(a->k_strides[0], a->B) || broadcast(a->v_strides[0], a->B) ||
        broadcast(a->k_strides[1], a->Hkv) || broadcast(a->v_strides[1], a->Hkv))
        return pl;
    if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o)) return pl;
    if (!tma_strides_ok({a->q_strides[2], a->q_strides[0] ? a->q_strides[0] : 8, a->k_strides[2],
                         a->k_strides[1] ? a->k_strides[1] : 8, a->k_strides[0] ? a->k_strides[0] : 8,
                         a->v_strides[2], a->v_strides[1] ? a->v_strides[1] : 8,
                         a->v_strides[0] ? a->v_strides[0] : 8}))
        return pl;
    for (int i = 0; i < 3; ++i)
        if ((a->o_strides[i] * 2) % 16) return pl;
    pl.path = Path::Tc;
    pl.n_tiles = (a->H / a->Hkv * a->Tq + kTcBM - 1) / kTcBM;
    pl.grid = pl.n_tiles * a->B * a->Hkv * pl.n_slices;
    pl.stages = tc_max_stages(a->D);
    if ((a->flags & ARC_FLAG_SINGLE_CTA) || !pair_supported(a->D, pl.dvs, false)) maybe_two(pl, a->D, false, a->B * a->Hkv);
    if (!pl.two && !(a->flags & ARC_FLAG_SINGLE_CTA) && pair_supported(a->D, pl.dvs, false)) {
        pl.pair = true;
        pl.stages = pair_max_stages(a->D);
        // persistent: at most one resident cluster per two SMs walks the list of row-tile pairs
        const int items = ((pl.n_tiles + 1) / 2) * a->B * a->Hkv;
        pl.grid = 2 * std::min(items, std::max(1, sm_count() / 2));
    }
    return pl;
}

SimpleParams simple_from_attn(const arc_attn_args *a)
{
    SimpleParams p{};
    p.mode = 0;
    p.dtype = a->dtype;
    p.B = a->B, p.H = a->H, p.Hkv = a->Hkv, p.Tq = a->Tq, p.Tk = a->Tk, p.Dqk = a->D, p.Dv = a->Dv, p.Dn = a->D;
    p.q = a->q, p.k = a->k, p.v = a->v, p.o = a->o;
    for (int i = 0; i < 3; ++i) p.qs[i] = a->q_strides[i], p.ks[i] = a->k_strides[i], p.vs[i] = a->v_strides[i],
                                p.os[i] = a->o_strides[i];
    p.lse = a->lse, p.sinks = a->sinks, p.scale = call_scale(a->flags, a->scale, a->D), p.causal = a->causal;
    p.status = a->status;
    return p;
}

// ------------------------------------------------------------------ MLA

arc_status check_mla(const arc_mla_args *a)
{
    if (!a) return ARC_ERR_INVALID_ARG;
    if (a->B < 0 || a->H <= 0 || a->Tq < 0 || a->Tk < 0 || a->Dn <= 0 || a->Dr < 0 || a->Dv <= 0)
        return ARC_ERR_INVALID_ARG;
    if (a->Dn + a->Dr > 512 || a->Dv > 512) return ARC_ERR_UNSUPPORTED;
    if (a->B == 0 || a->Tq == 0) return ARC_OK;
    if (!scale_ok(a->flags, a->scale)) return ARC_ERR_INVALID_ARG;
    if (!a->q_nope || (a->Dr > 0 && !a->q_rope) || !a->o || !a->lse) return ARC_ERR_INVALID_ARG;
    if (a->Tk > 0 && (!a->k_nope || (a->Dr > 0 && !a->k_rope) || !a->v)) return ARC_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        if (a->q_nope_strides[i] < 0 || a->q_rope_strides[i] < 0 || a->k_nope_strides[i] < 0 || a->v_strides[i] < 0 ||
            a->o_strides[i] < 0 || (i < 2 && a->k_rope_strides[i] < 0))
            return ARC_ERR_INVALID_ARG;
    if (broadcast(a->o_strides[0], a->B) || broadcast(a->o_strides[1], a->H) || broadcast(a->o_strides[2], a->Tq))
        return ARC_ERR_INVALID_ARG;
    return ARC_OK;
}

AttnPlan plan_mla(const arc_mla_args *a)
{
    AttnPlan pl;
    if (a->B == 0 || a->Tq == 0) return pl;
    if ((a->flags & ARC_FLAG_FORCE_SIMPLE) || a->Tk == 0) {
        pl.path = Path::Simple;
        return pl;
    }
    const int dqk = a->Dn + a->Dr;
    if (a->Dn % 64 || a->Dr % 64 || a->Dr == 0 || a->Dv > 256 || !tc_pair_supported(dqk, a->Dv, true)) return pl;
    if (a->q_nope_strides[1] != (int64_t)a->Tq * a->q_nope_strides[2] && a->H > 1) return pl;
    if (a->q_rope_strides[1] != (int64_t)a->Tq * a->q_rope_strides[2] && a->H > 1) return pl;
    if (broadcast(a->q_nope_strides[0], a->B) || broadcast(a->q_rope_strides[0], a->B) ||
        broadcast(a->k_nope_strides[0], a->B) || broadcast(a->k_nope_strides[1], a->H) ||
        broadcast(a->k_rope_strides[0], a->B) || broadcast(a->v_strides[0], a->B) || broadcast(a->v_strides[1], a->H))
        return pl;
    if (!aligned16(a->q_nope) || !aligned16(a->q_rope) || !aligned16(a->k_nope) || !aligned16(a->k_rope) ||
        !aligned16(a->v) || !aligned16(a->o))
        return pl;
    auto nz = [](int64_t s) { return s ? s : (int64_t)8; };
    if (!tma_strides_ok({a->q_nope_strides[2], nz(a->q_nope_strides[0]), a->q_rope_strides[2],
                         nz(a->q_rope_strides[0]), a->k_nope_strides[2], nz(a->k_nope_strides[1]),
                         nz(a->k_nope_strides[0]), a->k_rope_strides[1], nz(a->k_rope_strides[0]),
                         a->v_strides[2], nz(a->v_strides[1]), nz(a->v_strides[0])}))
        return pl;
    for (int i = 0; i < 3; ++i)
        if ((a->o_strides[i] * 2) % 16) return pl;
    pl.path = Path::Tc;
    pl.dvs = a->Dv;
    pl.n_slices = 1;
    pl.n_tiles = (a->Tq + kTcBM - 1) / kTcBM;
    pl.grid = pl.n_tiles * a->B * a->H;
    pl.stages = tc_max_stages(dqk);
    maybe_two(pl, dqk, true, a->B * a->H);
    if (!(a->flags & ARC_FLAG_SINGLE_CTA) && pair_supported(dqk, a->Dv, true)) {
        // CTA pair (M = 256), persistent like the dense pair path
        pl.two = false;
        pl.pair = true;
        pl.stages = pair_max_stages(dqk);
        const int items = ((pl.n_tiles + 1) / 2) * a->B * a->H;
        pl.grid = 2 * std::min(items, std::max(1, sm_count() / 2));
    }
    return pl;
}

// ------------------------------------------------------------------ sparse

arc_status check_sparse(const arc_sparse_args *a)
{
    if (!a) return ARC_ERR_INVALID_ARG;
    if (a->Sq < 0 || a->H <= 0 || a->Skv < 0 || a->topk < 0 || a->Dqk <= 0 || a->Dv <= 0) return ARC_ERR_INVALID_ARG;
    if (a->Dqk > 512 || a->Dv > 512) return ARC_ERR_UNSUPPORTED;
    if (!a->v && a->Dv > a->Dqk) return ARC_ERR_INVALID_ARG;
    if (a->Sq == 0) return ARC_OK;
    if (!scale_ok(a->flags, a->scale)) return ARC_ERR_INVALID_ARG;
    if (!a->q || !a->o || !a->lse || (a->topk > 0 && (!a->idx || !a->kv))) return ARC_ERR_INVALID_ARG;
    if (a->q_strides[0] < 0 || a->q_strides[1] < 0 || a->o_strides[0] < 0 || a->o_strides[1] < 0 || a->kv_stride < 0 ||
        a->v_stride < 0 || a->idx_stride < 0)
        return ARC_ERR_INVALID_ARG;
    if (broadcast(a->o_strides[0], a->Sq) || broadcast(a->o_strides[1], a->H)) return ARC_ERR_INVALID_ARG;
    return ARC_OK;
}

// Tensor-core sparse path: instantiated head dims, 16-byte aligned rows.
bool plan_sparse_tc(const arc_sparse_args *a)
{
    if (a->flags & ARC_FLAG_FORCE_SIMPLE) return false;
    const bool sepv = a->v != nullptr;
    if (!sparse_tc_supported(a->Dqk, a->Dv, sepv)) return false;
    if (!aligned16(a->q) || !aligned16(a->kv) || !aligned16(a->o) || (sepv && !aligned16(a->v))) return false;
    auto al = [](int64_t s) { return (s * 2) % 16 == 0; };
    if (!al(a->q_strides[0]) || !al(a->q_strides[1]) || !al(a->kv_stride) || !al(a->o_strides[0]) ||
        !al(a->o_strides[1]) || (sepv && !al(a->v_stride)))
        return false;
    return true;
}

// Decode-shaped sparse calls: when the tokens' (token, head group) CTAs leave SMs idle,
// each token's slots are cut into `splits` chunks of whole 64-slot tiles (at least two
// tiles each, at most ARC_MERGE_MAX_PARTS chunks), merged afterwards by the LSE merge.
struct SparseDecodePlan {
    bool tc = false;    // the tensor-core kernel takes the call
    int splits = 1, chunk = 0;
    size_t ws = 0;      // fp32 partials: O [splits][Sq][H][Dv] then LSE [splits][Sq][H]
};

SparseDecodePlan plan_sparse_decode(const arc_sparse_args *a)
{
    SparseDecodePlan pl;
    pl.chunk = std::max(1, a->topk);
    if (a->Sq == 0 || !plan_sparse_tc(a)) return pl;
    pl.tc = true;
    // the merge writes rows r = token * H + head at r * Dv: O must be [Sq, H, Dv] contiguous
    if (a->o_strides[1] != a->Dv || a->o_strides[0] != (int64_t)a->H * a->Dv) return pl;
    const int base = a->Sq * ((a->H + 63) / 64);
    const int tiles = (a->topk + 63) / 64;
    int splits = std::min({ARC_MERGE_MAX_PARTS, sm_count() / std::max(1, base), tiles / 2});
    if (splits < 2) return pl;
    const int chunk = ((tiles + splits - 1) / splits) * 64;
    splits = (a->topk + chunk - 1) / chunk;
    if (splits < 2) return pl;
    pl.splits = splits;
    pl.chunk = chunk;
    pl.ws = (size_t)splits * a->Sq * a->H * (a->Dv + 1) * sizeof(float);
    return pl;
}

// ------------------------------------------------------------------ backward

arc_status check_bwd(const arc_attn_bwd_args *a)
{
    if (!a) return ARC_ERR_INVALID_ARG;
    if (a->B < 0 || a->H <= 0 || a->Hkv <= 0 || a->H % a->Hkv || a->Tq < 0 || a->Tk < 0 || a->D <= 0 || a->Dv <= 0)
        return ARC_ERR_INVALID_ARG;
    if (!bwd_supported(a->D, a->Dv)) return ARC_ERR_UNSUPPORTED;
    if (a->B == 0 || a->Tq == 0) return ARC_OK;
    if (!scale_ok(a->flags, a->scale)) return ARC_ERR_INVALID_ARG;
    if (!a->q || !a->o || !a->dout || !a->lse || !a->dq || (a->Tk > 0 && (!a->k || !a->v || !a->dk || !a->dv)))
        return ARC_ERR_INVALID_ARG;
    if (a->sinks && !a->dsinks) return ARC_ERR_INVALID_ARG;
    const int64_t *all[] = {a->q_strides, a->k_strides, a->v_strides, a->o_strides, a->do_strides,
                            a->dq_strides, a->dk_strides, a->dv_strides};
    for (const int64_t *st : all)
        for (int i = 0; i < 3; ++i)
            if (st[i] < 0) return ARC_ERR_INVALID_ARG;
    // outputs whose rows would alias one another
    if (broadcast(a->dq_strides[0], a->B) || broadcast(a->dq_strides[1], a->H) || broadcast(a->dq_strides[2], a->Tq) ||
        broadcast(a->dk_strides[0], a->B) || broadcast(a->dk_strides[1], a->Hkv) || broadcast(a->dk_strides[2], a->Tk) ||
        broadcast(a->dv_strides[0], a->B) || broadcast(a->dv_strides[1], a->Hkv) || broadcast(a->dv_strides[2], a->Tk))
        return ARC_ERR_INVALID_ARG;
    // the tensor-core layout: fold rows evenly spaced, 16-byte rows and bases
    if (a->H > 1 && (a->q_strides[1] != (int64_t)a->Tq * a->q_strides[2] ||
                     a->do_strides[1] != (int64_t)a->Tq * a->do_strides[2]))
        return ARC_ERR_UNSUPPORTED;
    const void *ptrs[] = {a->q, a->k, a->v, a->o, a->dout, a->dq, a->dk, a->dv};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return ARC_ERR_UNSUPPORTED;
    for (const int64_t *st : all)
        for (int i = 0; i < 3; ++i)
            if ((st[i] * 2) % 16) return ARC_ERR_UNSUPPORTED;
    if (broadcast(a->q_strides[0], a->B) || broadcast(a->k_strides[0], a->B) || broadcast(a->v_strides[0], a->B) ||
        broadcast(a->k_strides[1], a->Hkv) || broadcast(a->v_strides[1], a->Hkv) || broadcast(a->do_strides[0], a->B))
        return ARC_ERR_UNSUPPORTED;
    return ARC_OK;
}

struct BwdPlan {
    int rsplit = 1, tiles_per_split = 0, n_kt = 0, n_qt = 0;
    size_t delta_bytes = 0, ws = 0;
};

// dK/dV: one CTA per (batch, kv head, key tile); when those are fewer than two per SM,
// each key tile's fold rows are split over several CTAs (at least 4 fold tiles each,
// about two CTAs per SM in all) whose fp32 partials a reduction sums.  More, smaller
// CTAs also even out the causal mask's uneven work per key tile.
BwdPlan plan_bwd(const arc_attn_bwd_args *a)
{
    BwdPlan pl;
    pl.delta_bytes = (((size_t)a->B * a->H * a->Tq * sizeof(float)) + 255) / 256 * 256;
    pl.ws = pl.delta_bytes;
    if (a->B == 0 || a->Tq == 0 || a->Tk == 0) return pl;
    const int BR = bwd_tile_rows(a->D, a->Dv);
    pl.n_kt = (a->Tk + 127) / 128;
    pl.n_qt = (a->H / a->Hkv * a->Tq + BR - 1) / BR;
    const int base = a->B * a->Hkv * pl.n_kt;
    const int want = 2 * sm_count();
    int rsplit = base >= want ? 1 : std::min((want + base - 1) / base, pl.n_qt / 4);
    rsplit = std::max(1, std::min(rsplit, 64));
    pl.tiles_per_split = (pl.n_qt + rsplit - 1) / rsplit;
    pl.rsplit = (pl.n_qt + pl.tiles_per_split - 1) / pl.tiles_per_split;
    if (pl.rsplit > 1)
        pl.ws += (size_t)pl.rsplit * a->B * a->Hkv * a->Tk * (a->D + a->Dv) * sizeof(float);
    return pl;
}

// ------------------------------------------------------------------ decode

struct DecodePlan {
    bool simple = false;
    bool tma = false;   // shape allows the TMA ring (cell stride a multiple of 16 bytes)
    int mf = 1;         // m16 fragments of fold rows per CTA
    int row_groups = 1; // CTAs along the fold rows of one (sequence, kv head)
    int splits = 0, chunk = 0, max_kv = 0, max_rows = 0;
    size_t ws = 0;
};

arc_status check_decode(const arc_decode_args *a, bool need_ptrs = true)
{
    if (!a) return ARC_ERR_INVALID_ARG;
    if (a->kv_type != ARC_KV_Q8_0 && a->kv_type != ARC_KV_Q4_0) return ARC_ERR_INVALID_ARG;
    if (a->n_tok < 0 || a->H <= 0 || a->Hkv <= 0 || a->H % a->Hkv || a->n_cells < 0 || a->n_seq < 0)
        return ARC_ERR_INVALID_ARG;
    if (a->n_seq > ARC_DECODE_MAX_SEQ) return ARC_ERR_UNSUPPORTED;
    if (!in_set(a->D, {64, 128, 256, 512})) return ARC_ERR_UNSUPPORTED;
    if (a->n_seq > 0 && !a->seqs) return ARC_ERR_INVALID_ARG;
    const int G = a->H / a->Hkv;
    for (int s = 0; s < a->n_seq; ++s) {
        const arc_seq &q = a->seqs[s];
        if (q.n_q < 0 || q.n_kv < q.n_q || q.q_begin < 0 || q.kv_begin < 0) return ARC_ERR_INVALID_ARG;
        if ((int64_t)q.q_begin + q.n_q > a->n_tok || (int64_t)q.kv_begin + q.n_kv > a->n_cells)
            return ARC_ERR_INVALID_ARG;
        if (G * q.n_q > ARC_DECODE_MAX_ROWS) return ARC_ERR_UNSUPPORTED;
    }
    if (need_ptrs && a->n_seq > 0 && a->n_tok > 0) {
        if (!scale_ok(a->flags, a->scale)) return ARC_ERR_INVALID_ARG;
        if (!a->q || !a->o || !a->lse || !a->k_cache || !a->v_cache) return ARC_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(a->k_cache) | reinterpret_cast<uintptr_t>(a->v_cache)) & 7u)
            return ARC_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(a->q) | reinterpret_cast<uintptr_t>(a->o)) & 7u) return ARC_ERR_INVALID_ARG;
    }
    return ARC_OK;
}

DecodePlan plan_decode(const arc_decode_args *a)
{
    DecodePlan pl;
    const int G = a->H / a->Hkv;
    for (int s = 0; s < a->n_seq; ++s) {
        pl.max_kv = std::max(pl.max_kv, a->seqs[s].n_kv);
        pl.max_rows = std::max(pl.max_rows, G * a->seqs[s].n_q);
    }
    const int64_t cell_bytes = (int64_t)a->Hkv * (a->D / 32) * (a->kv_type == ARC_KV_Q8_0 ? 34 : 18);
    pl.tma = cell_bytes % 16 == 0;
    // The split kernels: the TMA one for every head dim and up to ARC_DECODE_MAX_ROWS fold
    // rows (row groups of 16 or 32); the cp.async one (cell strides that are not 16-byte
    // multiples) for D <= 128 and one 16-row fragment.  Everything else, and
    // ARC_FLAG_FORCE_SIMPLE, runs the CUDA-core kernel.
    pl.simple = (a->flags & ARC_FLAG_FORCE_SIMPLE) != 0 || (!pl.tma && (a->D > 128 || pl.max_rows > 16));
    if (pl.simple || pl.max_kv == 0) return pl;
    pl.mf = (pl.max_rows > 16 && decode_ws_supported(a->kv_type, a->D, 2) && pl.tma) ? 2 : 1;
    pl.row_groups = (pl.max_rows + 16 * pl.mf - 1) / (16 * pl.mf);
    const int pairs = a->n_seq * a->Hkv * pl.row_groups;
    // One wave: as many CTAs as the SMs hold at once.  The occupancy API counts
    // registers as well as shared memory (the warp-specialised kernel is register-
    // limited to 3 CTAs per SM even where its stages would leave room for a fourth);
    // without a device, the shared-memory estimate.
    const int smem = decode_smem_bytes(a->kv_type, a->D, pl.mf, pl.tma);
    const int occ = decode_blocks_per_sm(a->kv_type, a->D, pl.mf, pl.tma);
    const int per_sm = occ > 0 ? std::min(4, occ) : std::max(1, std::min(4, (228 * 1024) / (smem + 1024)));
    const int target = sm_count() * per_sm;
    int splits = std::min(256, std::max(1, target / std::max(1, pairs)));
    int chunk = (pl.max_kv + splits - 1) / splits;
    chunk = ((chunk + 127) / 128) * 128;
    splits = (pl.max_kv + chunk - 1) / chunk;
    pl.splits = splits;
    pl.chunk = chunk;
    pl.ws = (size_t)pairs * splits * 16 * pl.mf * (a->D + 2) * sizeof(float);
    return pl;
}

}  // namespace

// ====================================================================== ABI

extern "C" {

int32_t arc_abi_version(void) { return ARC_ABI_VERSION; }

const char *arc_status_string(arc_status s)
{
    switch (s) {
    case ARC_OK: return "ok";
    case ARC_ERR_INVALID_ARG: return "invalid argument";
    case ARC_ERR_UNSUPPORTED: return "unsupported shape or layout";
    case ARC_ERR_CUDA: return "CUDA error";
    case ARC_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case ARC_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

arc_status arc_attn_fwd(const arc_attn_args *a, void *stream)
{
    arc_status st = check_attn(a);
    if (st != ARC_OK) return st;
    if (a->B == 0 || a->Tq == 0) return ARC_OK;
    AttnPlan pl = plan_attn(a);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pl.path == Path::None) return ARC_ERR_UNSUPPORTED;
    cudaError_t e;
    if (pl.path == Path::Simple) {
        note_dispatch("simple_attn_kernel");
        e = launch_simple_attn(simple_from_attn(a), s);
    } else {
        TcParams p;
        memset(&p, 0, sizeof(p));
        const uint64_t qd[3] = {(uint64_t)a->D, (uint64_t)a->H * a->Tq, (uint64_t)a->B};
        const int64_t qs[2] = {a->q_strides[2], a->q_strides[0] ? a->q_strides[0] : (int64_t)a->H * a->Tq * a->q_strides[2]};
        const uint64_t kd[4] = {(uint64_t)a->D, (uint64_t)a->Tk, (uint64_t)a->Hkv, (uint64_t)a->B};
        const int64_t ks[3] = {a->k_strides[2], a->k_strides[1] ? a->k_strides[1] : (int64_t)a->Tk * a->k_strides[2],
                               a->k_strides[0] ? a->k_strides[0] : (int64_t)a->Hkv * a->Tk * a->k_strides[2]};
        const uint64_t vd[4] = {(uint64_t)a->Dv, (uint64_t)a->Tk, (uint64_t)a->Hkv, (uint64_t)a->B};
        const int64_t vs[3] = {a->v_strides[2], a->v_strides[1] ? a->v_strides[1] : (int64_t)a->Tk * a->v_strides[2],
                               a->v_strides[0] ? a->v_strides[0] : (int64_t)a->Hkv * a->Tk * a->v_strides[2]};
        const uint32_t kv_box = pl.pair ? 64 : kTcBN;  // a CTA of a pair stages half of each key tile
        const int G = a->H / a->Hkv;
        // The pair kernel visits the fold rows of a kv head t-major (row = t*G + head in group)
        // when G divides the 128-row box: a tile then spans 128/G positions of every head of
        // the group, so under the causal mask all its rows need nearly the same key tiles.
        p.tmajor = pl.pair && G > 1 && kTcBM % G == 0;
        bool ok_q;
        if (p.tmajor) {
            const int64_t hs = a->q_strides[1] ? a->q_strides[1] : (int64_t)a->Tq * a->q_strides[2];
            const uint64_t qd5[5] = {(uint64_t)a->D, (uint64_t)G, (uint64_t)a->Tq, (uint64_t)a->Hkv, (uint64_t)a->B};
            const int64_t qs5[4] = {hs, a->q_strides[2], hs * G, qs[1]};
            const uint32_t box5[5] = {64, (uint32_t)G, (uint32_t)(kTcBM / G), 1, 1};
            ok_q = make_map_box(&p.tm_q, a->q, 5, qd5, qs5, box5);
        } else {
            ok_q = make_map(&p.tm_q, a->q, 3, qd, qs, kTcBM);
        }
        if (!ok_q || !make_map(&p.tm_k, a->k, 4, kd, ks, kv_box) || !make_map(&p.tm_v, a->v, 4, vd, vs, kv_box))
            return ARC_ERR_CUDA;
        p.tm_q2 = p.tm_q;
        p.tm_k2 = p.tm_k;
        p.B = a->B, p.H = a->H, p.Hkv = a->Hkv, p.G = a->H / a->Hkv, p.Tq = a->Tq, p.Tk = a->Tk, p.Dv = a->Dv;
        p.n_tiles = pl.n_tiles, p.n_slices = pl.n_slices, p.kc_first = a->D / 64, p.stages = pl.stages;
        p.o = a->o;
        for (int i = 0; i < 3; ++i) p.os[i] = a->o_strides[i];
        p.lse = a->lse, p.sinks = a->sinks, p.scale_log2 = call_scale(a->flags, a->scale, a->D) * kLog2e;
        p.causal = a->causal;
        p.status = a->status;
        if (pl.two) {
            order_tiles(p, (pl.n_tiles + 1) / 2, 2 * kTcBM);
            note_dispatch("tc_attn2_kernel");
            e = launch_tc_attn2(p, a->D, pl.dvs, false, pl.grid, s);
        } else if (pl.pair) {
            order_tiles(p, (pl.n_tiles + 1) / 2, 2 * kTcBM);
            note_dispatch("tc_attn_pair_kernel");
            e = launch_tc_attn_pair(p, a->D, pl.dvs, false, pl.grid, s);
        } else {
            order_tiles(p, pl.n_tiles);
            note_dispatch("tc_attn_kernel");
            e = launch_tc_attn(p, a->D, pl.dvs, false, pl.grid, s);
        }
    }
    return e == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

arc_status arc_mla_fwd(const arc_mla_args *a, void *stream)
{
    arc_status st = check_mla(a);
    if (st != ARC_OK) return st;
    if (a->B == 0 || a->Tq == 0) return ARC_OK;
    AttnPlan pl = plan_mla(a);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pl.path == Path::None) return ARC_ERR_UNSUPPORTED;
    cudaError_t e;
    if (pl.path == Path::Simple) {
        SimpleParams p{};
        p.mode = 1;
        p.dtype = ARC_DTYPE_BF16;
        p.B = a->B, p.H = a->H, p.Hkv = a->H, p.Tq = a->Tq, p.Tk = a->Tk, p.Dqk = a->Dn + a->Dr, p.Dv = a->Dv;
        p.Dn = a->Dn;
        p.q = a->q_nope, p.q2 = a->q_rope, p.k = a->k_nope, p.k2 = a->k_rope, p.v = a->v, p.o = a->o;
        for (int i = 0; i < 3; ++i) {
            p.qs[i] = a->q_nope_strides[i], p.q2s[i] = a->q_rope_strides[i], p.ks[i] = a->k_nope_strides[i];
            p.vs[i] = a->v_strides[i], p.os[i] = a->o_strides[i];
        }
        p.k2s[0] = a->k_rope_strides[0], p.k2s[1] = a->k_rope_strides[1];
        p.lse = a->lse, p.scale = call_scale(a->flags, a->scale, a->Dn + a->Dr), p.causal = a->causal;
        p.status = a->status;
        note_dispatch("simple_attn_kernel");
        e = launch_simple_attn(p, s);
    } else {
        TcParams p;
        memset(&p, 0, sizeof(p));
        auto nz = [](int64_t s_, int64_t dflt) { return s_ ? s_ : dflt; };
        const uint64_t qnd[3] = {(uint64_t)a->Dn, (uint64_t)a->H * a->Tq, (uint64_t)a->B};
        const int64_t qns[2] = {a->q_nope_strides[2], nz(a->q_nope_strides[0], (int64_t)a->H * a->Tq * a->q_nope_strides[2])};
        const uint64_t qrd[3] = {(uint64_t)a->Dr, (uint64_t)a->H * a->Tq, (uint64_t)a->B};
        const int64_t qrs[2] = {a->q_rope_strides[2], nz(a->q_rope_strides[0], (int64_t)a->H * a->Tq * a->q_rope_strides[2])};
        const uint64_t knd[4] = {(uint64_t)a->Dn, (uint64_t)a->Tk, (uint64_t)a->H, (uint64_t)a->B};
        const int64_t kns[3] = {a->k_nope_strides[2], nz(a->k_nope_strides[1], (int64_t)a->Tk * a->k_nope_strides[2]),
                                nz(a->k_nope_strides[0], (int64_t)a->H * a->Tk * a->k_nope_strides[2])};
        const uint64_t krd[3] = {(uint64_t)a->Dr, (uint64_t)a->Tk, (uint64_t)a->B};
        const int64_t krs[2] = {a->k_rope_strides[1], nz(a->k_rope_strides[0], (int64_t)a->Tk * a->k_rope_strides[1])};
        const uint64_t vd[4] = {(uint64_t)a->Dv, (uint64_t)a->Tk, (uint64_t)a->H, (uint64_t)a->B};
        const int64_t vs[3] = {a->v_strides[2], nz(a->v_strides[1], (int64_t)a->Tk * a->v_strides[2]),
                               nz(a->v_strides[0], (int64_t)a->H * a->Tk * a->v_strides[2])};
        const uint32_t kv_box = pl.pair ? 64 : kTcBN;   // a CTA of a pair stages half of each key tile
        if (!make_map(&p.tm_q, a->q_nope, 3, qnd, qns, kTcBM) || !make_map(&p.tm_q2, a->q_rope, 3, qrd, qrs, kTcBM) ||
            !make_map(&p.tm_k, a->k_nope, 4, knd, kns, kv_box) || !make_map(&p.tm_k2, a->k_rope, 3, krd, krs, kv_box) ||
            !make_map(&p.tm_v, a->v, 4, vd, vs, kv_box))
            return ARC_ERR_CUDA;
        p.B = a->B, p.H = a->H, p.Hkv = a->H, p.G = 1, p.Tq = a->Tq, p.Tk = a->Tk, p.Dv = a->Dv;
        p.n_tiles = pl.n_tiles, p.n_slices = 1, p.kc_first = a->Dn / 64, p.stages = pl.stages;
        p.o = a->o;
        for (int i = 0; i < 3; ++i) p.os[i] = a->o_strides[i];
        p.lse = a->lse, p.sinks = nullptr, p.scale_log2 = call_scale(a->flags, a->scale, a->Dn + a->Dr) * kLog2e;
        p.causal = a->causal;
        p.status = a->status;
        if (pl.pair) {
            order_tiles(p, (pl.n_tiles + 1) / 2, 2 * kTcBM);
            note_dispatch("tc_attn_pair_kernel<mla>");
            e = launch_tc_attn_pair(p, a->Dn + a->Dr, a->Dv, true, pl.grid, s);
        } else if (pl.two) {
            order_tiles(p, (pl.n_tiles + 1) / 2, 2 * kTcBM);
            note_dispatch("tc_attn2_kernel<mla>");
            e = launch_tc_attn2(p, a->Dn + a->Dr, a->Dv, true, pl.grid, s);
        } else {
            order_tiles(p, pl.n_tiles);
            note_dispatch("tc_attn_kernel<mla>");
            e = launch_tc_attn(p, a->Dn + a->Dr, a->Dv, true, pl.grid, s);
        }
    }
    return e == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

arc_status arc_sparse_mla_fwd(const arc_sparse_args *a, void *stream)
{
    arc_status st = check_sparse(a);
    if (st != ARC_OK) return st;
    if (a->Sq == 0) return ARC_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (plan_sparse_tc(a)) {
        SparseTcParams p{};
        p.Sq = a->Sq, p.H = a->H, p.Skv = a->Skv, p.Dqk = a->Dqk, p.Dv = a->Dv, p.topk = a->topk;
        p.q = static_cast<const __nv_bfloat16 *>(a->q), p.qs[0] = a->q_strides[0], p.qs[1] = a->q_strides[1];
        p.kv = static_cast<const __nv_bfloat16 *>(a->kv), p.kv_stride = a->kv_stride;
        p.v = static_cast<const __nv_bfloat16 *>(a->v), p.v_stride = a->v_stride;
        p.idx = a->idx, p.idx_stride = a->idx_stride;
        p.o = static_cast<__nv_bfloat16 *>(a->o), p.os[0] = a->o_strides[0], p.os[1] = a->o_strides[1];
        p.lse = a->lse, p.sinks = a->sinks, p.scale_log2 = call_scale(a->flags, a->scale, a->Dqk) * kLog2e;
        p.status = a->status;
        p.splits = 1, p.chunk = std::max(1, a->topk);
        note_dispatch("sparse_tc_kernel");
        e = launch_sparse_tc(p, s);
    } else {
        SimpleParams p{};
        p.mode = 2;
        p.dtype = ARC_DTYPE_BF16;
        p.B = 1, p.H = a->H, p.Hkv = 1, p.Tq = a->Sq, p.Tk = a->topk, p.Dqk = a->Dqk, p.Dv = a->Dv, p.Dn = a->Dqk;
        p.q = a->q, p.k = a->kv, p.v = a->v, p.o = a->o;
        p.qs[0] = a->q_strides[0], p.qs[1] = a->q_strides[1];
        p.ks[0] = a->kv_stride, p.vs[0] = a->v_stride;
        p.os[0] = a->o_strides[0], p.os[1] = a->o_strides[1];
        p.lse = a->lse, p.sinks = a->sinks, p.scale = call_scale(a->flags, a->scale, a->Dqk), p.causal = 0;
        p.idx = a->idx, p.idx_stride = a->idx_stride, p.topk = a->topk, p.Skv = a->Skv, p.status = a->status;
        note_dispatch("simple_attn_kernel<sparse>");
        e = launch_simple_attn(p, s);
    }
    return e == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

size_t arc_attn_bwd_workspace_size(const arc_attn_bwd_args *a)
{
    if (check_bwd(a) != ARC_OK) return 0;
    return plan_bwd(a).ws;
}

}  // extern "C"

namespace {

// The MLA extras of a backward call: q = q_nope || q_rope and k = k_nope || k_rope, the
// rope part of k one tensor shared by every head (its gradient is summed over them).
struct MlaBwdExtra {
    int Dn = 0, Dr = 0;
    const void *q_rope = nullptr;
    const int64_t *q_rope_strides = nullptr;
    const void *k_rope = nullptr;
    const int64_t *k_rope_strides = nullptr;
    void *dq_rope = nullptr;
    const int64_t *dq_rope_strides = nullptr;
    void *dk_rope = nullptr;
    const int64_t *dk_rope_strides = nullptr;
};

size_t mla_rope_part_bytes(const arc_attn_bwd_args *a, const BwdPlan &pl, int Dr)
{
    return (size_t)pl.rsplit * a->B * a->H * a->Tk * Dr * sizeof(float);
}

// Both backward calls after validation: delta (and the sink gradient), then dK / dV and
// dQ.  `a` is the call seen as dense attention over the concatenated head dims (for MLA:
// q and k are the nope tensors, D = Dn + Dr, Hkv = H); `mla` is non-null for MLA.
arc_status run_bwd(const arc_attn_bwd_args *a, const MlaBwdExtra *mla, void *workspace, size_t ws_bytes,
                   cudaStream_t s)
{
    const BwdPlan pl = plan_bwd(a);
    const size_t need = pl.ws + (mla ? mla_rope_part_bytes(a, pl, mla->Dr) : 0);
    if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return ARC_ERR_WORKSPACE;
    const float scale = call_scale(a->flags, a->scale, a->D);
    float *delta = static_cast<float *>(workspace);
    BwdPrepParams pp{};
    pp.B = a->B, pp.H = a->H, pp.Tq = a->Tq, pp.Dv = a->Dv;
    pp.o = static_cast<const __nv_bfloat16 *>(a->o), pp.dout = static_cast<const __nv_bfloat16 *>(a->dout);
    for (int i = 0; i < 3; ++i) pp.os[i] = a->o_strides[i], pp.dos[i] = a->do_strides[i];
    pp.lse = a->lse, pp.dlse = a->dlse, pp.sinks = a->sinks, pp.delta = delta, pp.dsinks = a->dsinks;
    note_dispatch("bwd_prep_kernel");
    if (launch_bwd_prep(pp, s) != cudaSuccess) return ARC_ERR_CUDA;

    BwdParams p;
    memset(&p, 0, sizeof(p));
    const int G = a->H / a->Hkv;
    const int BR = bwd_tile_rows(a->D, a->Dv);
    const int dn = mla ? mla->Dn : a->D;                     // columns of q / k in the first tensor
    auto qmap = [&](CUtensorMap *m, const void *base, const int64_t *st3, int width, uint32_t rows) {
        const uint64_t d[3] = {(uint64_t)width, (uint64_t)a->H * a->Tq, (uint64_t)a->B};
        const int64_t sv[2] = {st3[2], st3[0] ? st3[0] : (int64_t)a->H * a->Tq * st3[2]};
        return make_map(m, base, 3, d, sv, rows);
    };
    auto kmap = [&](CUtensorMap *m, const void *base, const int64_t *st3, int width) {
        const uint64_t d[4] = {(uint64_t)width, (uint64_t)a->Tk, (uint64_t)a->Hkv, (uint64_t)a->B};
        const int64_t sv[3] = {st3[2], st3[1] ? st3[1] : (int64_t)a->Tk * st3[2],
                               st3[0] ? st3[0] : (int64_t)a->Hkv * a->Tk * st3[2]};
        return make_map(m, base, 4, d, sv, 128);
    };
    if (a->Tk > 0 &&
        (!qmap(&p.tm_q, a->q, a->q_strides, dn, 128) || !qmap(&p.tm_do, a->dout, a->do_strides, a->Dv, 128) ||
         !qmap(&p.tm_qr, a->q, a->q_strides, dn, BR) || !qmap(&p.tm_dor, a->dout, a->do_strides, a->Dv, BR) ||
         !kmap(&p.tm_k, a->k, a->k_strides, dn) || !kmap(&p.tm_v, a->v, a->v_strides, a->Dv)))
        return ARC_ERR_CUDA;
    if (mla && a->Tk > 0) {
        const uint64_t kd[3] = {(uint64_t)mla->Dr, (uint64_t)a->Tk, (uint64_t)a->B};
        const int64_t *kr = mla->k_rope_strides;
        const int64_t ks[2] = {kr[1], kr[0] ? kr[0] : (int64_t)a->Tk * kr[1]};
        if (!qmap(&p.tm_q2, mla->q_rope, mla->q_rope_strides, mla->Dr, 128) ||
            !qmap(&p.tm_qr2, mla->q_rope, mla->q_rope_strides, mla->Dr, BR) || !make_map(&p.tm_k2, mla->k_rope, 3, kd, ks, 128))
            return ARC_ERR_CUDA;
    }
    p.mla = mla != nullptr, p.kc_first = dn / 64;
    p.B = a->B, p.H = a->H, p.Hkv = a->Hkv, p.G = G, p.Tq = a->Tq, p.Tk = a->Tk, p.D = a->D, p.Dv = a->Dv;
    p.causal = a->causal;
    p.lse = a->lse, p.delta = delta;
    p.scale = scale, p.scale_log2 = scale * kLog2e;
    p.dq = static_cast<__nv_bfloat16 *>(a->dq), p.dk = static_cast<__nv_bfloat16 *>(a->dk);
    p.dv = static_cast<__nv_bfloat16 *>(a->dv);
    for (int i = 0; i < 3; ++i) p.dqs[i] = a->dq_strides[i], p.dks[i] = a->dk_strides[i], p.dvs[i] = a->dv_strides[i];
    p.dk_cols = dn;
    if (mla) {
        p.dq2 = static_cast<__nv_bfloat16 *>(mla->dq_rope);
        for (int i = 0; i < 3; ++i) p.dq2s[i] = mla->dq_rope_strides[i];
        p.dk2 = static_cast<__nv_bfloat16 *>(mla->dk_rope);
        p.dk2s[0] = mla->dk_rope_strides[0], p.dk2s[1] = mla->dk_rope_strides[1];
        p.dkr_part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + pl.ws);
    }
    p.rsplit = pl.rsplit, p.tiles_per_split = pl.tiles_per_split;
    p.dkv_part = pl.rsplit > 1 ? reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + pl.delta_bytes) : nullptr;
    p.status = a->status;
    if (a->Tk == 0) p.rsplit = 1;   // no key: every gradient is zero; the dQ kernel writes dQ
    // dQ tiles by decreasing causal work (key tiles visible to the tile's last position),
    // so the heaviest go out first; without a mask every tile is alike
    const int n_rt = (G * a->Tq + 127) / 128;
    if (a->causal && n_rt <= 1024) {
        const int n_kt = (a->Tk + 127) / 128;
        std::vector<std::pair<int, int>> w(n_rt);
        for (int rt = 0; rt < n_rt; ++rt) {
            const int r0 = rt * 128, rl = std::min(r0 + 128, G * a->Tq) - 1;
            const int t_max = (r0 / a->Tq != rl / a->Tq) ? a->Tq - 1 : rl % a->Tq;
            const int nk = std::max(0, std::min(a->Tk, t_max + a->Tk - a->Tq + 1));
            w[rt] = {-std::min(n_kt, (nk + 127) / 128), rt};
        }
        std::stable_sort(w.begin(), w.end());
        p.dq_order_n = n_rt;
        for (int i = 0; i < n_rt; ++i) p.dq_order[i] = (uint16_t)w[i].second;
    }
    note_dispatch(mla ? "bwd_dkdv_kernel<mla>" : "bwd_dkdv_kernel");
    note_dispatch("bwd_dq_kernel");
    return launch_bwd(p, s) == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

// An MLA backward call as dense attention over the concatenated head dims (Hkv = H, the
// nope tensors as q and k), for the shared checks, the plan and the launch.
arc_attn_bwd_args mla_as_dense(const arc_mla_bwd_args *m)
{
    arc_attn_bwd_args a;
    memset(&a, 0, sizeof(a));
    a.B = m->B, a.H = m->H, a.Hkv = m->H, a.Tq = m->Tq, a.Tk = m->Tk, a.D = m->Dn + m->Dr, a.Dv = m->Dv;
    a.q = m->q_nope, a.k = m->k_nope, a.v = m->v, a.o = m->o, a.dout = m->dout;
    a.dq = m->dq_nope, a.dk = m->dk_nope, a.dv = m->dv;
    for (int i = 0; i < 3; ++i) {
        a.q_strides[i] = m->q_nope_strides[i], a.k_strides[i] = m->k_nope_strides[i], a.v_strides[i] = m->v_strides[i];
        a.o_strides[i] = m->o_strides[i], a.do_strides[i] = m->do_strides[i];
        a.dq_strides[i] = m->dq_nope_strides[i], a.dk_strides[i] = m->dk_nope_strides[i];
        a.dv_strides[i] = m->dv_strides[i];
    }
    a.lse = m->lse, a.dlse = m->dlse;
    a.scale = m->scale, a.causal = m->causal, a.flags = m->flags, a.status = m->status;
    return a;
}

arc_status check_mla_bwd(const arc_mla_bwd_args *m)
{
    if (!m) return ARC_ERR_INVALID_ARG;
    if (m->Dn <= 0 || m->Dr <= 0 || m->Dn % 64 || m->Dr % 64) return ARC_ERR_UNSUPPORTED;
    const arc_attn_bwd_args a = mla_as_dense(m);
    arc_status st = check_bwd(&a);
    if (st != ARC_OK || m->B == 0 || m->Tq == 0) return st;
    if (!m->q_rope || !m->dq_rope || (m->Tk > 0 && (!m->k_rope || !m->dk_rope))) return ARC_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        if (m->q_rope_strides[i] < 0 || m->dq_rope_strides[i] < 0 || (i < 2 && (m->k_rope_strides[i] < 0 || m->dk_rope_strides[i] < 0)))
            return ARC_ERR_INVALID_ARG;
    if (broadcast(m->dq_rope_strides[0], m->B) || broadcast(m->dq_rope_strides[1], m->H) ||
        broadcast(m->dq_rope_strides[2], m->Tq) || broadcast(m->dk_rope_strides[0], m->B) ||
        broadcast(m->dk_rope_strides[1], m->Tk))
        return ARC_ERR_INVALID_ARG;
    if (m->H > 1 && m->q_rope_strides[1] != (int64_t)m->Tq * m->q_rope_strides[2]) return ARC_ERR_UNSUPPORTED;
    const void *ptrs[] = {m->q_rope, m->k_rope, m->dq_rope, m->dk_rope};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return ARC_ERR_UNSUPPORTED;
    for (int i = 0; i < 3; ++i)
        if ((m->q_rope_strides[i] * 2) % 16 || (m->dq_rope_strides[i] * 2) % 16 ||
            (i < 2 && ((m->k_rope_strides[i] * 2) % 16 || (m->dk_rope_strides[i] * 2) % 16)))
            return ARC_ERR_UNSUPPORTED;
    if (broadcast(m->q_rope_strides[0], m->B) || broadcast(m->k_rope_strides[0], m->B)) return ARC_ERR_UNSUPPORTED;
    return ARC_OK;
}

MlaBwdExtra mla_extra(const arc_mla_bwd_args *m)
{
    MlaBwdExtra x;
    x.Dn = m->Dn, x.Dr = m->Dr;
    x.q_rope = m->q_rope, x.q_rope_strides = m->q_rope_strides;
    x.k_rope = m->k_rope, x.k_rope_strides = m->k_rope_strides;
    x.dq_rope = m->dq_rope, x.dq_rope_strides = m->dq_rope_strides;
    x.dk_rope = m->dk_rope, x.dk_rope_strides = m->dk_rope_strides;
    return x;
}

}  // namespace

extern "C" {

arc_status arc_attn_bwd(const arc_attn_bwd_args *a, void *workspace, size_t ws_bytes, void *stream)
{
    arc_status st = check_bwd(a);
    if (st != ARC_OK) return st;
    if (a->B == 0 || a->Tq == 0) return ARC_OK;
    return run_bwd(a, nullptr, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t arc_mla_bwd_workspace_size(const arc_mla_bwd_args *m)
{
    if (check_mla_bwd(m) != ARC_OK) return 0;
    const arc_attn_bwd_args a = mla_as_dense(m);
    const BwdPlan pl = plan_bwd(&a);
    return pl.ws + mla_rope_part_bytes(&a, pl, m->Dr);
}

arc_status arc_mla_bwd(const arc_mla_bwd_args *m, void *workspace, size_t ws_bytes, void *stream)
{
    arc_status st = check_mla_bwd(m);
    if (st != ARC_OK) return st;
    if (m->B == 0 || m->Tq == 0) return ARC_OK;
    const arc_attn_bwd_args a = mla_as_dense(m);
    const MlaBwdExtra x = mla_extra(m);
    return run_bwd(&a, &x, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t arc_sparse_decode_workspace_size(const arc_sparse_args *a)
{
    if (check_sparse(a) != ARC_OK) return 0;
    return plan_sparse_decode(a).ws;
}

arc_status arc_sparse_mla_decode(const arc_sparse_args *a, void *workspace, size_t ws_bytes, void *stream)
{
    arc_status st = check_sparse(a);
    if (st != ARC_OK) return st;
    if (a->Sq == 0) return ARC_OK;
    const SparseDecodePlan pl = plan_sparse_decode(a);
    if (pl.splits == 1) return arc_sparse_mla_fwd(a, stream);
    if (!workspace || ws_bytes < pl.ws || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return ARC_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SparseTcParams p{};
    p.Sq = a->Sq, p.H = a->H, p.Skv = a->Skv, p.Dqk = a->Dqk, p.Dv = a->Dv, p.topk = a->topk;
    p.q = static_cast<const __nv_bfloat16 *>(a->q), p.qs[0] = a->q_strides[0], p.qs[1] = a->q_strides[1];
    p.kv = static_cast<const __nv_bfloat16 *>(a->kv), p.kv_stride = a->kv_stride;
    p.v = static_cast<const __nv_bfloat16 *>(a->v), p.v_stride = a->v_stride;
    p.idx = a->idx, p.idx_stride = a->idx_stride;
    p.o = static_cast<__nv_bfloat16 *>(a->o), p.os[0] = a->o_strides[0], p.os[1] = a->o_strides[1];
    p.lse = a->lse, p.sinks = a->sinks, p.scale_log2 = call_scale(a->flags, a->scale, a->Dqk) * kLog2e;
    p.status = a->status;
    p.splits = pl.splits, p.chunk = pl.chunk;
    const size_t rows = (size_t)a->Sq * a->H;
    p.part_o = static_cast<float *>(workspace);
    p.part_lse = p.part_o + (size_t)pl.splits * rows * a->Dv;
    note_dispatch("sparse_tc_kernel<split>");
    if (launch_sparse_tc(p, s) != cudaSuccess) return ARC_ERR_CUDA;
    // LSE merge of the splits (and the sink, once), fp32 partials into the bf16 output
    MergeParams m{};
    m.n_parts = pl.splits, m.rows = (int)rows, m.dv = a->Dv, m.dtype = ARC_DTYPE_F32, m.out_dtype = ARC_DTYPE_BF16;
    for (int i = 0; i < pl.splits; ++i) {
        m.o_parts[i] = p.part_o + (size_t)i * rows * a->Dv;
        m.lse_parts[i] = p.part_lse + (size_t)i * rows;
    }
    m.sinks = a->sinks, m.sink_heads = a->H, m.sink_rows = 1;
    m.o = a->o, m.lse = a->lse;
    return launch_merge(m, s) == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

size_t arc_decode_workspace_size(const arc_decode_args *a)
{
    if (check_decode(a, false) != ARC_OK) return 0;
    return plan_decode(a).ws;
}

arc_status arc_attn_decode_q8(const arc_decode_args *a, void *workspace, size_t ws_bytes, void *stream)
{
    arc_status st = check_decode(a);
    if (st != ARC_OK) return st;
    if (a->n_seq == 0 || a->n_tok == 0) return ARC_OK;
    DecodePlan pl = plan_decode(a);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (pl.simple || pl.max_kv == 0) {
        SimpleDecodeParams p{};
        p.kv_type = a->kv_type, p.n_tok = a->n_tok, p.H = a->H, p.Hkv = a->Hkv, p.D = a->D;
        p.n_cells = a->n_cells, p.n_seq = a->n_seq;
        p.q = a->q, p.k_cache = static_cast<const uint8_t *>(a->k_cache);
        p.v_cache = static_cast<const uint8_t *>(a->v_cache);
        memcpy(p.seqs, a->seqs, sizeof(arc_seq) * a->n_seq);
        p.o = a->o, p.lse = a->lse, p.scale = call_scale(a->flags, a->scale, a->D);
        note_dispatch("simple_decode_kernel");
        e = launch_simple_decode(p, s);
    } else {
        if (!workspace || ws_bytes < pl.ws || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return ARC_ERR_WORKSPACE;
        DecodeParams p{};
        p.kv_type = a->kv_type, p.n_tok = a->n_tok, p.H = a->H, p.Hkv = a->Hkv, p.D = a->D, p.n_seq = a->n_seq;
        p.splits = pl.splits, p.chunk = pl.chunk;
        p.mf = pl.mf, p.rows = 16 * pl.mf, p.row_groups = pl.row_groups;
        p.q = a->q, p.k_cache = static_cast<const uint8_t *>(a->k_cache);
        p.v_cache = static_cast<const uint8_t *>(a->v_cache);
        memcpy(p.seqs, a->seqs, sizeof(arc_seq) * a->n_seq);
        p.o = a->o, p.lse = a->lse;
        const size_t parts = (size_t)a->n_seq * a->Hkv * pl.row_groups * pl.splits;
        p.ws_o = static_cast<float *>(workspace);
        p.ws_ml = p.ws_o + parts * p.rows * a->D;
        p.scale_log2 = call_scale(a->flags, a->scale, a->D) * kLog2e;
        p.status = a->status;
        // K/V tiles by TMA when the cache rows allow it: a byte tensor {cell bytes, n_cells} per cache.
        p.tma = pl.tma && (reinterpret_cast<uintptr_t>(a->k_cache) & 15) == 0 &&
                (reinterpret_cast<uintptr_t>(a->v_cache) & 15) == 0;
        if (p.tma) {
            const int64_t cell_bytes = (int64_t)a->Hkv * (a->D / 32) * (a->kv_type == ARC_KV_Q8_0 ? 34 : 18);
            int box_w = 0, box_cells = 0;
            decode_box(a->kv_type, a->D, pl.mf, &box_w, &box_cells);
            if (box_w <= 0 ||
                !make_map_bytes_cached(&p.tm_kc, a->k_cache, (uint64_t)cell_bytes, (uint64_t)a->n_cells, box_w, box_cells) ||
                !make_map_bytes_cached(&p.tm_vc, a->v_cache, (uint64_t)cell_bytes, (uint64_t)a->n_cells, box_w, box_cells))
                return ARC_ERR_CUDA;
            note_dispatch(a->kv_type == ARC_KV_Q8_0 ? "decode_ws_kernel<q8_0>" : "decode_ws_kernel<q4_0>");
        } else if (a->D <= 128 && pl.max_rows <= 16) {
            note_dispatch(a->kv_type == ARC_KV_Q8_0 ? "decode_split_kernel<q8_0>" : "decode_split_kernel<q4_0>");
        } else {
            // the shape allows TMA but these caches are not 16-byte aligned: the CUDA-core kernel
            SimpleDecodeParams q{};
            q.kv_type = a->kv_type, q.n_tok = a->n_tok, q.H = a->H, q.Hkv = a->Hkv, q.D = a->D;
            q.n_cells = a->n_cells, q.n_seq = a->n_seq;
            q.q = a->q, q.k_cache = static_cast<const uint8_t *>(a->k_cache);
            q.v_cache = static_cast<const uint8_t *>(a->v_cache);
            memcpy(q.seqs, a->seqs, sizeof(arc_seq) * a->n_seq);
            q.o = a->o, q.lse = a->lse, q.scale = call_scale(a->flags, a->scale, a->D);
            note_dispatch("simple_decode_kernel");
            return launch_simple_decode(q, s) == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
        }
        e = launch_decode(p, s);
    }
    return e == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

// Library-owned scratch for arc_attn_decode_q8_noalloc.  In host code the
// symbol is only a stand-in; its device address comes from
// cudaGetSymbolAddress, looked up with the caller's context current.
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[ARC_DECODE_NOALLOC_SCRATCH_BYTES];

// Identity of the calling thread's current CUDA context, unique for the life of the
// process (a context re-created after cudaDeviceReset gets a new one), or 0 when
// there is no current context or the driver cannot say.
static unsigned long long current_context_id()
{
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// The scratch array's device address in the current context.  The symbol can sit at a
// different address in every context that loads the library (another device, a context
// made current through the driver API, the primary context re-created after a reset), so
// the address is cached per context id, never per device ordinal.  Without an id the
// lookup runs on every call.
static arc_status noalloc_scratch_address(void **out)
{
    struct Entry {
        unsigned long long ctx;
        void *addr;
    };
    static std::mutex mu;
    static Entry cache[64];
    static int used = 0, next = 0;
    std::lock_guard<std::mutex> lock(mu);
    unsigned long long id = current_context_id();
    for (int i = 0; id && i < used; ++i)
        if (cache[i].ctx == id) {
            *out = cache[i].addr;
            return ARC_OK;
        }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return ARC_ERR_CUDA;
    }
    if (!id) id = current_context_id();   // the lookup may have made the primary context current
    if (id) {
        cache[next] = {id, p};
        next = (next + 1) % 64;
        used = std::max(used, next == 0 ? 64 : next);
    }
    *out = p;
    return ARC_OK;
}

arc_status arc_attn_decode_q8_noalloc(const arc_decode_args *a, void *stream)
{
    arc_status st = check_decode(a);
    if (st != ARC_OK) return st;
    if (a->n_seq == 0 || a->n_tok == 0) return ARC_OK;
    if (plan_decode(a).ws > ARC_DECODE_NOALLOC_SCRATCH_BYTES) return ARC_ERR_WORKSPACE;
    void *scratch = nullptr;
    if ((st = noalloc_scratch_address(&scratch)) != ARC_OK) return st;
    return arc_attn_decode_q8(a, scratch, ARC_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}

static arc_status check_merge(const arc_merge_args *a)
{
    if (!a) return ARC_ERR_INVALID_ARG;
    if (a->n_parts < 1 || a->n_parts > ARC_MERGE_MAX_PARTS || a->rows < 0 || a->dv <= 0 || (a->dv & 1))
        return ARC_ERR_INVALID_ARG;
    if (a->dv > 1024) return ARC_ERR_UNSUPPORTED;
    if (a->dtype != ARC_DTYPE_F32 && a->dtype != ARC_DTYPE_BF16) return ARC_ERR_INVALID_ARG;
    if (a->sinks && (a->sink_heads <= 0 || a->sink_rows <= 0)) return ARC_ERR_INVALID_ARG;
    if (a->rows == 0) return ARC_OK;
    auto bad = [](const void *ptr) { return !ptr || (reinterpret_cast<uintptr_t>(ptr) & 7u); };
    if (bad(a->o) || bad(a->lse)) return ARC_ERR_INVALID_ARG;
    for (int i = 0; i < a->n_parts; ++i)
        if (bad(a->o_parts[i]) || !a->lse_parts[i] || (reinterpret_cast<uintptr_t>(a->lse_parts[i]) & 3u))
            return ARC_ERR_INVALID_ARG;
    return ARC_OK;
}

arc_status arc_attn_merge(const arc_merge_args *a, void *stream)
{
    const arc_status st = check_merge(a);
    if (st != ARC_OK || a->rows == 0) return st;
    MergeParams p{};
    p.n_parts = a->n_parts, p.rows = a->rows, p.dv = a->dv, p.dtype = a->dtype, p.out_dtype = a->dtype;
    for (int i = 0; i < a->n_parts; ++i) p.o_parts[i] = a->o_parts[i], p.lse_parts[i] = a->lse_parts[i];
    p.sinks = a->sinks, p.sink_heads = a->sink_heads, p.sink_rows = a->sink_rows;
    p.o = a->o, p.lse = a->lse;
    note_dispatch("merge_kernel");
    return launch_merge(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

arc_status arc_plan(int32_t op, const void *args, arc_plan_info *out)
{
    if (!args || !out) return ARC_ERR_INVALID_ARG;
    if (op == ARC_OP_ATTN) {
        const arc_attn_args *a = static_cast<const arc_attn_args *>(args);
        arc_status st = check_attn(a);
        if (st != ARC_OK) return st;
        AttnPlan pl = plan_attn(a);
        if (a->B == 0 || a->Tq == 0) {
            set_name(out, "none");
            return ARC_OK;
        }
        if (pl.path == Path::None) return ARC_ERR_UNSUPPORTED;
        if (pl.path == Path::Simple) {
            set_name(out, "simple_attn_kernel");
            out->tile_m = 4;
            out->n_ctas = (int)(((int64_t)a->B * a->H * a->Tq + 3) / 4);
        } else {
            set_name(out, pl.two ? "tc_attn2_kernel" : (pl.pair ? "tc_attn_pair_kernel" : "tc_attn_kernel"));
            out->tensor_cores = 1;
            out->tile_m = (pl.two || pl.pair) ? 2 * kTcBM : kTcBM, out->tile_n = kTcBN, out->d_slice = pl.dvs;
            out->n_ctas = pl.grid;
            out->smem_bytes = pl.two ? tc2_smem_bytes(a->D, pl.stages)
                                     : (pl.pair ? pair_smem_bytes(a->D, pl.stages) : tc_smem_bytes(a->D, pl.stages));
            out->tmem_cols = 512;
        }
        out->launches = 1;
        return ARC_OK;
    }
    if (op == ARC_OP_MLA) {
        const arc_mla_args *a = static_cast<const arc_mla_args *>(args);
        arc_status st = check_mla(a);
        if (st != ARC_OK) return st;
        AttnPlan pl = plan_mla(a);
        if (a->B == 0 || a->Tq == 0) {
            set_name(out, "none");
            return ARC_OK;
        }
        if (pl.path == Path::None) return ARC_ERR_UNSUPPORTED;
        if (pl.path == Path::Simple) {
            set_name(out, "simple_attn_kernel");
            out->tile_m = 4;
        } else {
            set_name(out, pl.pair ? "tc_attn_pair_kernel<mla>" : (pl.two ? "tc_attn2_kernel<mla>" : "tc_attn_kernel<mla>"));
            out->tensor_cores = 1;
            out->tile_m = (pl.two || pl.pair) ? 2 * kTcBM : kTcBM, out->tile_n = kTcBN, out->d_slice = pl.dvs,
            out->n_ctas = pl.grid;
            out->smem_bytes = pl.pair ? pair_smem_bytes(a->Dn + a->Dr, pl.stages)
                                      : (pl.two ? tc2_smem_bytes(a->Dn + a->Dr, pl.stages)
                                                : tc_smem_bytes(a->Dn + a->Dr, pl.stages));
            out->tmem_cols = 512;
        }
        out->launches = 1;
        return ARC_OK;
    }
    if (op == ARC_OP_MERGE) {
        const arc_merge_args *a = static_cast<const arc_merge_args *>(args);
        arc_status st = check_merge(a);
        if (st != ARC_OK) return st;
        set_name(out, "merge_kernel");
        out->n_ctas = (a->rows + 7) / 8;
        out->launches = a->rows > 0 ? 1 : 0;
        return ARC_OK;
    }
    if (op == ARC_OP_SPARSE) {
        const arc_sparse_args *a = static_cast<const arc_sparse_args *>(args);
        arc_status st = check_sparse(a);
        if (st != ARC_OK) return st;
        if (a->Sq > 0 && plan_sparse_tc(a)) {
            set_name(out, "sparse_tc_kernel");
            out->tensor_cores = 1;
            out->tile_m = 64, out->tile_n = 64, out->d_slice = a->Dv;
            out->n_ctas = a->Sq * ((a->H + 63) / 64);
            out->smem_bytes = sparse_smem_bytes(a->Dqk, a->Dv, a->v != nullptr), out->tmem_cols = 512;
        } else {
            set_name(out, "simple_attn_kernel<sparse>");
            out->tile_m = 4;
        }
        out->launches = 1;
        return ARC_OK;
    }
    if (op == ARC_OP_ATTN_BWD) {
        const arc_attn_bwd_args *a = static_cast<const arc_attn_bwd_args *>(args);
        arc_status st = check_bwd(a);
        if (st != ARC_OK) return st;
        if (a->B == 0 || a->Tq == 0) {
            set_name(out, "none");
            return ARC_OK;
        }
        const BwdPlan pl = plan_bwd(a);
        set_name(out, "bwd_dkdv_kernel+bwd_dq_kernel");
        out->tensor_cores = 1;
        out->tile_m = 128, out->tile_n = bwd_tile_rows(a->D, a->Dv), out->d_slice = a->D;
        out->splits = pl.rsplit;
        out->n_ctas = a->B * a->Hkv * pl.n_kt * pl.rsplit;
        out->smem_bytes = bwd_dkdv_smem_bytes(a->D, a->Dv), out->tmem_cols = 512;
        out->launches = 3 + (a->sinks ? 1 : 0) + (pl.rsplit > 1 ? 1 : 0);
        return ARC_OK;
    }
    if (op == ARC_OP_MLA_BWD) {
        const arc_mla_bwd_args *m = static_cast<const arc_mla_bwd_args *>(args);
        arc_status st = check_mla_bwd(m);
        if (st != ARC_OK) return st;
        if (m->B == 0 || m->Tq == 0) {
            set_name(out, "none");
            return ARC_OK;
        }
        const arc_attn_bwd_args a = mla_as_dense(m);
        const BwdPlan pl = plan_bwd(&a);
        set_name(out, "bwd_dkdv_kernel<mla>+bwd_dq_kernel");
        out->tensor_cores = 1;
        out->tile_m = 128, out->tile_n = bwd_tile_rows(a.D, a.Dv), out->d_slice = a.D;
        out->splits = pl.rsplit;
        out->n_ctas = a.B * a.Hkv * pl.n_kt * pl.rsplit;
        out->smem_bytes = bwd_dkdv_smem_bytes(a.D, a.Dv), out->tmem_cols = 512;
        out->launches = 4 + (pl.rsplit > 1 ? 1 : 0);
        return ARC_OK;
    }
    if (op == ARC_OP_SPARSE_DECODE) {
        const arc_sparse_args *a = static_cast<const arc_sparse_args *>(args);
        arc_status st = check_sparse(a);
        if (st != ARC_OK) return st;
        const SparseDecodePlan pl = plan_sparse_decode(a);
        if (a->Sq == 0) {
            set_name(out, "none");
            return ARC_OK;
        }
        if (!pl.tc) {
            set_name(out, "simple_attn_kernel<sparse>");
            out->tile_m = 4;
            out->launches = 1;
            return ARC_OK;
        }
        set_name(out, pl.splits > 1 ? "sparse_tc_kernel<split>" : "sparse_tc_kernel");
        out->tensor_cores = 1;
        out->tile_m = 64, out->tile_n = 64, out->d_slice = a->Dv;
        out->splits = pl.splits;
        out->n_ctas = a->Sq * ((a->H + 63) / 64) * pl.splits;
        out->smem_bytes = sparse_smem_bytes(a->Dqk, a->Dv, a->v != nullptr), out->tmem_cols = 512;
        out->launches = pl.splits > 1 ? 2 : 1;
        return ARC_OK;
    }
    if (op == ARC_OP_DECODE) {
        const arc_decode_args *a = static_cast<const arc_decode_args *>(args);
        arc_status st = check_decode(a);
        if (st != ARC_OK) return st;
        DecodePlan pl = plan_decode(a);
        if (pl.simple || pl.max_kv == 0) {
            set_name(out, "simple_decode_kernel");
            out->launches = 1;
        } else {
            // the TMA kernel needs 16-byte aligned caches; arc_plan reports the shape's choice
            const bool tma = pl.tma && (reinterpret_cast<uintptr_t>(a->k_cache) & 15) == 0 &&
                             (reinterpret_cast<uintptr_t>(a->v_cache) & 15) == 0;
            if (!tma && (a->D > 128 || pl.max_rows > 16)) {
                set_name(out, "simple_decode_kernel");
                out->launches = 1;
                return ARC_OK;
            }
            int box_w = 0, box_cells = 64;
            if (tma) {
                set_name(out, a->kv_type == ARC_KV_Q8_0 ? "decode_ws_kernel<q8_0>" : "decode_ws_kernel<q4_0>");
                decode_box(a->kv_type, a->D, pl.mf, &box_w, &box_cells);
            } else {
                set_name(out, a->kv_type == ARC_KV_Q8_0 ? "decode_split_kernel<q8_0>" : "decode_split_kernel<q4_0>");
            }
            out->tensor_cores = 1;
            // tile_m: fold rows per CTA; tile_n: cells per tile; d_slice: head dims one warp covers
            out->tile_m = 16 * pl.mf, out->tile_n = box_cells;
            out->d_slice = tma ? a->D / std::max(1, (a->D * pl.mf) / 128) : a->D;
            out->splits = pl.splits, out->n_ctas = a->n_seq * a->Hkv * pl.row_groups * pl.splits;
            out->smem_bytes = decode_smem_bytes(a->kv_type, a->D, pl.mf, tma);
            out->launches = 2;
        }
        return ARC_OK;
    }
    return ARC_ERR_INVALID_ARG;
}

arc_status arc_check_device_error(const uint32_t *status, void *stream)
{
    if (!status) return ARC_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ARC_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return ARC_ERR_CUDA;
    return v ? ARC_ERR_DEVICE_TIMEOUT : ARC_OK;
}

arc_status arc_selftest_timeout(uint32_t *status, uint64_t timeout_ns, void *stream)
{
    if (!status) return ARC_ERR_INVALID_ARG;
    return launch_selftest_timeout(status, timeout_ns, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? ARC_OK
               : ARC_ERR_CUDA;
}

}  // extern "C"
