// internal.h -- launch interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/arc_attn.h"

namespace arc {

// ---------------------------------------------------------------- CUDA-core kernels
// One warp per output row; lanes split the head dims; exact fp32 arithmetic.
// Used for fp32 "reference mode" and as the control arm (ARC_FLAG_FORCE_SIMPLE).
struct SimpleParams {
    int mode;  // 0 dense, 1 MLA, 2 sparse
    int dtype; // ARC_DTYPE_BF16 or ARC_DTYPE_F32
    int B, H, Hkv, Tq, Tk, Dqk, Dv, Dn;
    const void *q, *q2, *k, *k2, *v;
    int64_t qs[3], q2s[3], ks[3], k2s[3], vs[3], os[3];
    void *o;
    float *lse;
    const float *sinks;
    float scale;
    int causal;
    const int32_t *idx;
    int64_t idx_stride;
    int topk, Skv;
    uint32_t *status;
};
cudaError_t launch_simple_attn(const SimpleParams &p, cudaStream_t s);

struct SimpleDecodeParams {
    int kv_type, n_tok, H, Hkv, D, n_cells, n_seq;
    const float *q;
    const uint8_t *k_cache, *v_cache;
    arc_seq seqs[ARC_DECODE_MAX_SEQ];
    float *o, *lse;
    float scale;
};
cudaError_t launch_simple_decode(const SimpleDecodeParams &p, cudaStream_t s);

// ---------------------------------------------------------------- tcgen05 attention
// Dense / GQA fold / MLA forward, M = 128 query rows per CTA, K/V tiles by TMA.
struct TcParams {
    CUtensorMap tm_q;   // q (dense) or q_nope (MLA): dims {D, H*Tq, B}; t-major: {D, G, Tq, Hkv, B}
    CUtensorMap tm_q2;  // q_rope: dims {Dr, H*Tq, B}
    CUtensorMap tm_k;   // k (dense) or k_nope: dims {D, Tk, Hkv, B}
    CUtensorMap tm_k2;  // k_rope: dims {Dr, Tk, B}
    CUtensorMap tm_v;   // v: dims {Dv, Tk, Hkv, B}
    int B, H, Hkv, G, Tq, Tk, Dv;
    int n_tiles;        // query-row tiles per (b, kv) group
    int n_slices;       // d_v slices
    int kc_first;       // 64-column chunks of q/k taken from the first tensor (MLA: nope)
    int stages;         // ring stages
    void *o;
    int64_t os[3];
    float *lse;
    const float *sinks;
    float scale_log2;   // scale * log2(e)
    int causal;
    int tmajor;         // fold rows visited t-major (row = t*G + head-in-group); tm_q is then 5-d
    uint32_t *status;
    uint16_t tile_order[1024];
};
int tc_smem_bytes(int dqk, int stages);
int tc_max_stages(int dqk);
cudaError_t launch_tc_attn(const TcParams &p, int dqk, int dvs, bool mla, int grid, cudaStream_t s);
// Two query tiles per CTA sharing every K/V tile (d_v <= 128).
int tc2_smem_bytes(int dqk, int stages);
int tc2_max_stages(int dqk);
cudaError_t launch_tc_attn2(const TcParams &p, int dqk, int dvs, bool mla, int grid, cudaStream_t s);

// Pair of CTAs (cta_group::2, M = 256): dense d_qk in {256, 512} with a 256-wide
// d_v slice or d_qk in {128, 192, 256} with d_v 128; MLA d_qk 192 (128 + 64), d_v 128.
int pair_smem_bytes(int dqk, int stages);
int pair_max_stages(int dqk);
bool pair_supported(int dqk, int dvs, bool mla);
cudaError_t launch_tc_attn_pair(const TcParams &p, int dqk, int dvs, bool mla, int grid, cudaStream_t s);

// Sparse top-k forward, M = 64 heads of one query token per CTA, gathered rows.
struct SparseTcParams {
    int Sq, H, Skv, Dqk, Dv, topk;
    const __nv_bfloat16 *q;
    int64_t qs[2];
    const __nv_bfloat16 *kv;
    int64_t kv_stride;
    const __nv_bfloat16 *v;
    int64_t v_stride;
    const int32_t *idx;
    int64_t idx_stride;
    __nv_bfloat16 *o;
    int64_t os[2];
    float *lse;
    const float *sinks;
    float scale_log2;
    uint32_t *status;
    // Split top-k (decode-shaped calls): CTA (token, head group, split) takes slots
    // [split*chunk, min(topk, split*chunk + chunk)) and writes its normalised fp32 partial
    // O [splits][Sq][H][Dv] and LSE [splits][Sq][H] (no sink: the merge adds it).
    // splits == 1 and part_o == NULL: the whole list per CTA, bf16 O written directly.
    int splits, chunk;
    float *part_o, *part_lse;
};
int sparse_smem_bytes(int dqk, int dv, bool sepv);
bool sparse_tc_supported(int dqk, int dv, bool sepv);
cudaError_t launch_sparse_tc(const SparseTcParams &p, cudaStream_t s);

// ---------------------------------------------------------------- quantised decode
struct DecodeParams {
    CUtensorMap tm_kc;  // k_cache as bytes {Hkv*row bytes, n_cells}, box {slice span, tile cells} (tma != 0)
    CUtensorMap tm_vc;  // v_cache likewise
    int tma;            // 1: K/V tiles arrive by TMA through a multi-stage ring; 0: cp.async
    int kv_type, n_tok, H, Hkv, D, n_seq, splits, chunk;
    int mf;             // m16 fragments of fold rows per CTA (1 or 2)
    int rows;           // fold rows per CTA and per workspace part: 16 * mf
    int row_groups;     // CTAs along the fold rows of one (sequence, kv head)
    const float *q;
    const uint8_t *k_cache, *v_cache;
    arc_seq seqs[ARC_DECODE_MAX_SEQ];
    float *o, *lse;
    float *ws_o;     // [n_seq*Hkv*row_groups*splits][rows][D] partial outputs (unnormalised)
    float *ws_ml;    // [n_seq*Hkv*row_groups*splits][rows][2] partial (max, sum)
    float scale_log2;
    uint32_t *status;
};
cudaError_t launch_decode(const DecodeParams &p, cudaStream_t s);
// TMA split kernel instantiations: cache type x head dim (64..512) x fragments (1, 2; 1 at 512).
bool decode_ws_supported(int kv_type, int D, int mf);
int decode_smem_bytes(int kv_type, int D, int mf, bool tma);
int decode_blocks_per_sm(int kv_type, int D, int mf, bool tma);
void decode_box(int kv_type, int D, int mf, int *width, int *cells);

// ---------------------------------------------------------------- backward (dense / GQA, sinks)
// delta = rowsum(dO * O) - dLSE per row, and the sink gradient.
struct BwdPrepParams {
    int B, H, Tq, Dv;
    const __nv_bfloat16 *o, *dout;
    int64_t os[3], dos[3];
    const float *lse, *dlse, *sinks;
    float *delta;       // [B,H,Tq] (workspace)
    float *dsinks;      // [H]
};
cudaError_t launch_bwd_prep(const BwdPrepParams &p, cudaStream_t s);

struct BwdParams {
    CUtensorMap tm_q, tm_do;    // q / dO {D, H*Tq, B}, box {64, 128}      (dQ kernel)
    CUtensorMap tm_qr, tm_dor;  // the same, box {64, fold-tile rows}      (dK/dV kernel)
    CUtensorMap tm_k, tm_v;     // k / v {D, Tk, Hkv, B}, box {64, 128}
    // MLA: q = q_nope || q_rope and k = k_nope || k_rope (shared by the heads) are
    // concatenated on load; 64-column chunks from kc_first on come from the rope maps
    CUtensorMap tm_q2, tm_qr2;  // q_rope {Dr, H*Tq, B}, boxes {64, 128} and {64, fold-tile rows}
    CUtensorMap tm_k2;          // k_rope {Dr, Tk, B}, box {64, 128}
    int mla, kc_first;
    int B, H, Hkv, G, Tq, Tk, D, Dv;
    int causal;
    const float *lse, *delta;   // [B,H,Tq]
    float scale, scale_log2;
    __nv_bfloat16 *dq, *dk, *dv;
    int64_t dqs[3], dks[3], dvs[3];
    __nv_bfloat16 *dq2;         // MLA: dq_rope, strides dq2s; dq holds dq_nope
    int64_t dq2s[3];
    int dk_cols;                // columns of dK written to dk (D; MLA: Dn, the rope columns go to dkr_part)
    float *dkr_part;            // MLA: fp32 [rsplit][B][H][Tk][Dr] per-head rope columns of dK (unscaled)
    __nv_bfloat16 *dk2;         // MLA: dk_rope [B, Tk, Dr] (the sum over heads), strides dk2s
    int64_t dk2s[2];
    int rsplit, tiles_per_split;// dK/dV CTAs per key tile along the fold rows, and fold tiles each
    float *dkv_part;            // rsplit > 1: fp32 [rsplit][B][Hkv][Tk][D + Dv] (dK unscaled, then dV)
    uint32_t *status;
    // dQ CTAs go out rank by rank over all (batch, kv head) pairs; rank i takes fold tile
    // dq_order[i] (the tiles by decreasing causal work), or n_rt - 1 - i when dq_order_n is 0
    int dq_order_n;
    uint16_t dq_order[1024];
};
bool bwd_supported(int d, int dv);
int bwd_tile_rows(int d, int dv);
int bwd_dkdv_smem_bytes(int d, int dv);
int bwd_dq_smem_bytes(int d, int dv);
cudaError_t launch_bwd(const BwdParams &p, cudaStream_t s);

cudaError_t launch_selftest_timeout(uint32_t *status, uint64_t timeout_ns, cudaStream_t s);

// Merge of partial results over disjoint key sets (arc_attn_merge), one warp per row.
struct MergeParams {
    int n_parts, rows, dv, dtype;
    int out_dtype;      // dtype of o (the parts' dtype for arc_attn_merge; fp32 parts -> bf16 o for sparse decode)
    const void *o_parts[ARC_MERGE_MAX_PARTS];
    const float *lse_parts[ARC_MERGE_MAX_PARTS];
    const float *sinks;
    int sink_heads, sink_rows;
    void *o;
    float *lse;
};
cudaError_t launch_merge(const MergeParams &p, cudaStream_t s);

}  // namespace arc
