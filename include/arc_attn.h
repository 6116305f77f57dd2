/*
 * arc_attn.h -- C ABI of a fused exact-attention forward library for B200 (sm_100a).
 *
 * Every call computes, for each output row, exact softmax attention
 *
 *     O   = softmax(scale * q K^T + mask [+ sink]) V        (a row of d_v values)
 *     LSE = ln( sum_j exp(scale * q.k_j) [+ exp(sink)] )    (natural log, fp32)
 *
 * tiled over keys with an online softmax, so no score matrix is ever stored.
 * The forward output plus a per-row log-sum-exp is the output pair of the FA4
 * forward ("pith-train PR: FA4 b19 return arity", summary).  The arity of
 * every call is fixed by its argument struct; nothing is returned as a tuple
 * whose length could change between versions (the crash that page reports).
 *
 * Conventions shared by all calls
 *   - Pointers marked "device" are CUDA device (or managed) memory owned by the
 *     caller.  The library allocates no memory.  A call reads its inputs and
 *     writes its outputs (and, for decode, the caller's workspace), with two
 *     exceptions, both library-wide state: arc_attn_decode_q8_noalloc keeps its
 *     split-KV partials in one static device buffer that every call shares (see
 *     that call for its race and first-call-before-capture rules), and with
 *     ARC_LOG=1 in the environment the first launch of each kernel is noted on
 *     stderr (host-side bookkeeping that never changes a result).  Tensor maps
 *     for the decode caches are cached on the host, keyed by pointer and shape.
 *   - Strides are in ELEMENTS, int64.  The last dimension of every tensor is
 *     contiguous (stride 1).  A zero stride over a dimension of extent above 1
 *     (a broadcast view) is accepted for inputs by the CUDA-core kernels, which
 *     index it as given: the tensor-core attn / MLA paths cannot describe it in
 *     a TMA map and return ARC_ERR_UNSUPPORTED for it unless
 *     ARC_FLAG_FORCE_SIMPLE is set (the sparse gather reads it as given).  An
 *     output with such a stride (rows that alias) is ARC_ERR_INVALID_ARG.
 *   - `stream` is a cudaStream_t passed as void*.  NULL is the legacy default
 *     stream and is a valid stream.  Launches are asynchronous on it.
 *   - Arguments are validated on the host before anything is launched.  On
 *     ARC_ERR_INVALID_ARG / ARC_ERR_UNSUPPORTED nothing is launched and no
 *     output is written.  A failed launch returns ARC_ERR_CUDA.
 *   - `status` (optional, device, one uint32 the caller zeroes): every wait
 *     inside the kernels is bounded; a wait that runs out ORs a nonzero code
 *     into *status and the kernel returns early.  arc_check_device_error()
 *     reads it.  With status == NULL such an event is not reported.
 *   - Causal masks are bottom-right aligned: query i of Tq sees keys
 *     j <= i + (Tk - Tq).  A row with no visible key and no sink gets O = 0 and
 *     LSE = -inf.
 */
#ifndef ARC_ATTN_H
#define ARC_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ARC_ABI_VERSION 2

typedef enum {
    ARC_OK = 0,
    ARC_ERR_INVALID_ARG = 1,   /* a shape, pointer, stride or alignment is wrong */
    ARC_ERR_UNSUPPORTED = 2,   /* valid, but outside what the kernels implement */
    ARC_ERR_CUDA = 3,          /* a CUDA launch or runtime call failed */
    ARC_ERR_DEVICE_TIMEOUT = 4,/* a bounded device-side wait ran out (see status) */
    ARC_ERR_WORKSPACE = 5      /* workspace missing or smaller than required */
} arc_status;

typedef enum { ARC_DTYPE_BF16 = 0, ARC_DTYPE_F32 = 1 } arc_dtype;

/* Quantised KV block types; the values are the ggml type ids. */
typedef enum { ARC_KV_Q4_0 = 2, ARC_KV_Q8_0 = 8 } arc_kv_type;

typedef enum {
    ARC_OP_ATTN = 1, ARC_OP_MLA = 2, ARC_OP_SPARSE = 3, ARC_OP_DECODE = 4, ARC_OP_MERGE = 5,
    ARC_OP_SPARSE_DECODE = 6, ARC_OP_ATTN_BWD = 7, ARC_OP_MLA_BWD = 8
} arc_op;

/* flags (all calls) */
#define ARC_FLAG_FORCE_SIMPLE 1u   /* run the CUDA-core kernel instead of the tensor-core one */
#define ARC_FLAG_SINGLE_CTA 2u     /* do not use the CTA-pair (cta_group::2) kernel */
/* Use the standard softmax scale 1/sqrt(d_qk) and ignore the `scale` field:
 * d_qk is D (arc_attn_fwd, arc_attn_decode_q8), Dn + Dr (arc_mla_fwd) or Dqk
 * (arc_sparse_mla_fwd).  Without the flag, `scale` is used as given (any
 * finite value; NaN is ARC_ERR_INVALID_ARG). */
#define ARC_FLAG_DEFAULT_SCALE 4u

/* --------------------------------------------------------------------------
 * arc_attn_fwd: dense attention with GQA / MQA and optional per-head sinks.
 *
 * Source: "ArcFlash - Arc's own attention kernel, rung 0", section "What rung 0
 * does": query head h reads kv head h / g (g = H / Hkv; heads are kv-major, as
 * repeat_kv lays them out), and the GQA expansion is a reshape of q[B,H,Tq,D]
 * to [B,Hkv,g*Tq,D] with no copy of K or V; a sink is a per-head constant in
 * each row's softmax denominator and never multiplies V.
 *
 *   q  [B,H,Tq,D]     dtype, device, strides q_strides = {batch, head, token}
 *   k  [B,Hkv,Tk,D]   dtype, device
 *   v  [B,Hkv,Tk,Dv]  dtype, device
 *   o  [B,H,Tq,Dv]    dtype, device, written
 *   lse [B,H,Tq]      fp32, device, contiguous, written
 *   sinks [H]         fp32, device, or NULL for no sink; a raw logit (not scaled)
 *
 * dtype BF16: (D, Dv) in {(64,64), (128,64), (128,128), (192,128), (256,128),
 * (256,256), (256,512), (512,128), (512,256), (512,512)}; fp32 accumulation;
 * P is rounded to bf16 before P*V.  The tensor-core path needs
 * each (b, kv) group of g*Tq query rows evenly spaced (head stride ==
 * Tq * token stride), 16-byte aligned rows and base pointers; otherwise the
 * call returns ARC_ERR_UNSUPPORTED unless ARC_FLAG_FORCE_SIMPLE is set.
 * dtype F32 ("reference mode"): any D and Dv from 1 to 512, any strides;
 * CUDA-core fp32 arithmetic, no TF32.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t dtype;
    int32_t B, H, Hkv, Tq, Tk, D, Dv;
    const void *q; int64_t q_strides[3];
    const void *k; int64_t k_strides[3];
    const void *v; int64_t v_strides[3];
    void *o;       int64_t o_strides[3];
    float *lse;
    const float *sinks;
    float scale;
    int32_t causal;
    uint32_t flags;
    uint32_t *status;
} arc_attn_args;

arc_status arc_attn_fwd(const arc_attn_args *args, void *stream);

/* --------------------------------------------------------------------------
 * arc_mla_fwd: MLA attention with d_qk != d_v and the q/k concat done on load.
 *
 * Source: "pith-train PR: FA4 b19 return arity", MLA section: q = q_nope||q_rope
 * and k = k_nope||k_rope are concatenated and fed to the attention kernel with
 * head dims d_qk != d_v.  Here the concat is never materialised: the kernel
 * stages both parts of each row side by side.  k_rope is one tensor shared by
 * all heads.
 *
 *   q_nope [B,H,Tq,Dn]  bf16, device, strides {batch, head, token}
 *   q_rope [B,H,Tq,Dr]  bf16, device
 *   k_nope [B,H,Tk,Dn]  bf16, device
 *   k_rope [B,Tk,Dr]    bf16, device, strides {batch, token}
 *   v      [B,H,Tk,Dv]  bf16, device
 *   o      [B,H,Tq,Dv]  bf16, device, written
 *   lse    [B,H,Tq]     fp32, device, contiguous, written
 * Dn, Dr multiples of 64 (Dr > 0) with (Dn + Dr, Dv) in {(128,128), (192,64),
 * (192,128), (256,128), (256,256)}; 16-byte
 * aligned base pointers and strides, and each head's query rows evenly spaced
 * (head stride == Tq * token stride).  Other shapes or layouts return
 * ARC_ERR_UNSUPPORTED unless ARC_FLAG_FORCE_SIMPLE is set, which runs the
 * CUDA-core kernel for any Dn + Dr <= 512, Dv <= 512.  Dn + Dr or Dv above 512
 * is ARC_ERR_UNSUPPORTED; negative sizes or strides, or a NULL tensor that the
 * call reads, are ARC_ERR_INVALID_ARG.  B == 0 or Tq == 0 launches nothing.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t B, H, Tq, Tk, Dn, Dr, Dv;
    const void *q_nope; int64_t q_nope_strides[3];
    const void *q_rope; int64_t q_rope_strides[3];
    const void *k_nope; int64_t k_nope_strides[3];
    const void *k_rope; int64_t k_rope_strides[2];
    const void *v;      int64_t v_strides[3];
    void *o;            int64_t o_strides[3];
    float *lse;
    float scale;
    int32_t causal;
    uint32_t flags;
    uint32_t *status;
} arc_mla_args;

arc_status arc_mla_fwd(const arc_mla_args *args, void *stream);

/* --------------------------------------------------------------------------
 * arc_sparse_mla_fwd: attention over per-query top-k index lists.
 *
 * Source: "TensorRT-LLM: FlashMLA without -rdc", timing paragraph: sparse MLA
 * forward over 13312 queries x 64 heads x 2176 top-k at d_qk 512.  All heads of
 * a query token attend to the same gathered pool rows.  A slot whose index is
 * outside [0, Skv) (e.g. -1 padding) is masked; a repeated index counts once
 * per slot; no causal mask is applied (the index list encodes it).
 *
 *   q    [Sq,H,Dqk]   bf16, device, strides q_strides = {token, head}
 *   kv   [Skv,Dqk]    bf16, device, row stride kv_stride
 *   v    [Skv,Dv]     bf16, device, row stride v_stride; NULL means V is the
 *                     first Dv columns of the same kv row (an MLA latent)
 *   idx  [Sq,topk]    int32, device, row stride idx_stride
 *   o    [Sq,H,Dv]    bf16, device, strides o_strides = {token, head}, written
 *   lse  [Sq,H]       fp32, device, contiguous, written
 *   sinks [H]         fp32, device, or NULL
 * Dqk in {64,128,256,512}, Dv <= Dqk a multiple of 64.  The tensor-core
 * kernel takes (Dqk, Dv) = (512, 512), (512, 256), (256, 256), (128, 128) with
 * V inside the kv row, and (128, 64), (128, 128), (256, 256) with a separate v,
 * on 16-byte aligned base pointers and strides; every other supported call runs
 * the CUDA-core kernel (arc_plan names which).  Dqk or Dv above 512 is
 * ARC_ERR_UNSUPPORTED; negative sizes or strides, Dv > Dqk without v, or a
 * NULL tensor that the call reads are ARC_ERR_INVALID_ARG.  Sq == 0 launches
 * nothing.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t Sq, H, Skv, Dqk, Dv, topk;
    const void *q;      int64_t q_strides[2];
    const void *kv;     int64_t kv_stride;
    const void *v;      int64_t v_stride;
    const int32_t *idx; int64_t idx_stride;
    void *o;            int64_t o_strides[2];
    float *lse;
    const float *sinks;
    float scale;
    uint32_t flags;
    uint32_t *status;
} arc_sparse_args;

arc_status arc_sparse_mla_fwd(const arc_sparse_args *args, void *stream);

/* --------------------------------------------------------------------------
 * arc_sparse_mla_decode: the same sparse attention, shaped for decode batches.
 *
 * Source: "TensorRT-LLM: FlashMLA without -rdc", its ptxas list: next to the
 * sparse prefill, FlashMLA builds a sparse decode kernel for 64 heads ("sm100
 * sparse decode (h64)").  A decode batch has few query tokens, and
 * arc_sparse_mla_fwd runs one CTA per (token, 64-head group), which leaves most
 * SMs idle below ~148 tokens.  This call takes the same arguments and computes
 * the same O and LSE, but when the tokens do not fill the GPU it cuts each
 * token's top-k list into `splits` chunks of whole 64-slot tiles (one CTA each,
 * at most ARC_MERGE_MAX_PARTS), writes every chunk's normalised fp32 partial O
 * and LSE to the workspace, and merges them with the LSE-weighted output merge
 * of arc_attn_merge (the sink, if any, enters once, there): two launches.
 * When the tokens fill the GPU, or the call does not take the tensor-core
 * kernel, or o is not a contiguous [Sq,H,Dv] tensor, it is exactly
 * arc_sparse_mla_fwd (one launch, no workspace).
 *   workspace  device, at least arc_sparse_decode_workspace_size(args) bytes
 *              (0: none needed), 256-byte aligned, overwritten; its contents
 *              need no initialisation.  Two calls in flight need two.
 * Errors: those of arc_sparse_mla_fwd; a missing, short or unaligned workspace
 * where one is needed is ARC_ERR_WORKSPACE.  arc_plan(ARC_OP_SPARSE_DECODE)
 * names the kernel ("sparse_tc_kernel<split>" with the split count).
 * The fp8 KV variant the page also lists is an sm90 kernel; it is not built here
 * (the page gives no cache format for it).
 * ------------------------------------------------------------------------ */
size_t arc_sparse_decode_workspace_size(const arc_sparse_args *args);

arc_status arc_sparse_mla_decode(const arc_sparse_args *args, void *workspace, size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * arc_attn_decode_q8: multi-sequence decode over one unified q8_0 / q4_0 cache,
 * the K/V blocks dequantised in registers as each tile is loaded.
 *
 * Source: "unsloth llama.cpp: dequantize q4_0/q8_0 K/V tiles in the FA MMA
 * kernel", summary paragraph: with a q4_0 / q8_0 KV cache and 3 to 16 tokens per
 * batch across several sequences in one unified cache, K/V tiles are
 * dequantised as they are loaded instead of converting the whole cache first.
 *
 * Block formats (32 values plus an fp16 scale d, little endian, d first):
 *   q8_0: d, then 32 int8 q_j; value = d*q_j                          (34 bytes)
 *   q4_0: d, then 16 bytes, byte j = n_j | n_{j+16}<<4; value = d*(n-8) (18 bytes)
 *
 *   q        [n_tok,H,D]            fp32, device, contiguous
 *   k_cache  [n_cells,Hkv,D/32 blk] device, contiguous blocks, 8-byte aligned
 *   v_cache  same layout and type as k_cache
 *   seqs     [n_seq]                HOST array; sequence s owns query tokens
 *            q_begin..q_begin+n_q-1 and cells kv_begin..kv_begin+n_kv-1, and its
 *            n_q tokens are its last n_q cells: its token t (0-based) sees cells
 *            kv_begin .. kv_begin + n_kv - n_q + t.
 *   o        [n_tok,H,D]            fp32, device, written (rows of tokens that no
 *            sequence owns are left untouched)
 *   lse      [n_tok,H]              fp32, device, written likewise
 * D in {64,128,256,512}; H % Hkv == 0; (H/Hkv) * n_q <= ARC_DECODE_MAX_ROWS
 * for every sequence; n_seq <= ARC_DECODE_MAX_SEQ.  The query heads of a kv
 * head times a sequence's new tokens are its fold rows (row = head in group *
 * n_q + token).  On caches whose cell stride (Hkv * D/32 blocks) is a multiple
 * of 16 bytes and whose base pointers are 16-byte aligned, every head dim runs
 * the split-KV tensor-core kernel (TMA ring, m16n8k16 MMAs, 16 or 32 fold rows
 * per CTA, head dims above 128 cut into slices whose S partials are summed in
 * shared memory) and its combine: two launches.  Other caches run the cp.async
 * split kernel for D <= 128 with up to 16 fold rows, else the CUDA-core kernel
 * (one warp per query row over all its cells, one launch, no workspace), as
 * does ARC_FLAG_FORCE_SIMPLE.  arc_plan names the kernel.
 * workspace: device, at least arc_decode_workspace_size(args) bytes, 256-byte
 * aligned; used for the split-KV partial results and overwritten.  Its
 * contents need no initialisation (every byte read is first written by the
 * same call).  Two calls in flight at once need two workspaces.
 * Errors, all returned before anything is launched: D outside {64,128,256,512},
 * n_seq above ARC_DECODE_MAX_SEQ or (H/Hkv) * n_q above ARC_DECODE_MAX_ROWS is
 * ARC_ERR_UNSUPPORTED; an unknown kv_type, negative sizes, H % Hkv != 0,
 * n_kv < n_q, a sequence whose tokens or cells run past n_tok / n_cells, a NULL
 * tensor, or q, o or a cache not 8-byte aligned is ARC_ERR_INVALID_ARG; a
 * missing, short or unaligned workspace (where one is needed) is
 * ARC_ERR_WORKSPACE.  n_seq == 0 or n_tok == 0 launches nothing.
 * ------------------------------------------------------------------------ */
#define ARC_DECODE_MAX_SEQ 64
#define ARC_DECODE_MAX_ROWS 128

typedef struct {
    int32_t q_begin, n_q, kv_begin, n_kv;
} arc_seq;

typedef struct {
    int32_t kv_type;
    int32_t n_tok, H, Hkv, D, n_cells, n_seq;
    const float *q;
    const void *k_cache;
    const void *v_cache;
    const arc_seq *seqs;
    float *o;
    float *lse;
    float scale;
    uint32_t flags;
    uint32_t *status;
} arc_decode_args;

size_t arc_decode_workspace_size(const arc_decode_args *args);

arc_status arc_attn_decode_q8(const arc_decode_args *args, void *workspace, size_t ws_bytes,
                              void *stream);

/* --------------------------------------------------------------------------
 * arc_attn_decode_q8_noalloc: the same decode, for callers that cannot
 * allocate device memory.
 *
 * The pages have no counterpart to this call; it exists for hosts that must
 * not call cudaMalloc at all -- an engine whose memory planner owns every
 * device byte, a process that runs with a fixed memory budget, or code that
 * must stay out of the allocator while other work is in flight -- and so
 * cannot hand arc_attn_decode_q8 a workspace.  It takes the same arguments
 * minus the workspace and launches the same kernels, with the split-KV
 * partial results kept in a library-owned buffer: a file-scope __device__
 * array of ARC_DECODE_NOALLOC_SCRATCH_BYTES (8 MiB) that every GPU which loads
 * the library holds until the process exits.  The caller still passes all
 * inputs and outputs.
 *   - A call whose partial results would need more than that buffer returns
 *     ARC_ERR_WORKSPACE and launches nothing (arc_decode_workspace_size()
 *     gives the bytes a call needs).
 *   - The buffer's device address differs from context to context.  The first
 *     call in each CUDA context (the context current on the calling thread)
 *     looks it up with cudaGetSymbolAddress and keeps it, keyed by the
 *     context's unique id, so a context made current through the driver API or
 *     re-created after cudaDeviceReset gets its own lookup.  Make that first
 *     call before any stream capture.
 *   - All calls share the one buffer and it keeps the last call's contents
 *     (nothing in it needs to start at zero).  Calls that may overlap on the
 *     GPU -- on different streams without ordering between them -- race on it;
 *     serialise them.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 * ------------------------------------------------------------------------ */
#define ARC_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

arc_status arc_attn_decode_q8_noalloc(const arc_decode_args *args, void *stream);

/* --------------------------------------------------------------------------
 * arc_attn_merge: the exact result over a union of disjoint key sets, from
 * the results over each set.
 *
 * When the keys of every row are split over parts (context-parallel ranks,
 * or the chunks of a long sequence), each part gives its own normalised
 * output O_i and log-sum-exp LSE_i.  The merge is the output merge of
 * "TransformerEngine: FA4 in context-parallel attention" (flowchart):
 *
 *     LSE = ln( sum_i exp(LSE_i) [+ exp(sink)] )
 *     O   = sum_i exp(LSE_i - LSE) * O_i
 *
 * which equals attention over all the keys at once.  A per-head sink logit,
 * if given, is added once here (the parts must then be computed without it).
 * A part with LSE_i = -inf is empty and contributes nothing; a row whose
 * parts are all empty gets O = 0 and LSE = -inf (or = sink).
 *
 *   n_parts        1 .. ARC_MERGE_MAX_PARTS
 *   rows, dv       the parts and the output are [rows, dv], row stride dv
 *                  (a [B,H,Tq,Dv] output with contiguous rows is rows = B*H*Tq);
 *                  dv even, <= 1024
 *   dtype          arc_dtype of every O_i and of o (fp32 arithmetic inside)
 *   o_parts[i]     device, [rows, dv];   lse_parts[i]  device fp32, [rows]
 *   sinks          device fp32 or NULL; row r uses sinks[(r / sink_rows) % sink_heads]
 *                  (for [B,H,Tq] rows: sink_rows = Tq, sink_heads = H)
 *   o, lse         device, written: [rows, dv] and [rows] fp32
 * Pointers must be 8-byte aligned.  o may alias o_parts[0] and lse may alias
 * lse_parts[0] (each row is read in full before it is written).
 * ------------------------------------------------------------------------ */
#define ARC_MERGE_MAX_PARTS 16

typedef struct {
    int32_t n_parts, rows, dv, dtype;
    const void *o_parts[ARC_MERGE_MAX_PARTS];
    const float *lse_parts[ARC_MERGE_MAX_PARTS];
    const float *sinks;
    int32_t sink_heads, sink_rows;
    void *o;
    float *lse;
} arc_merge_args;

arc_status arc_attn_merge(const arc_merge_args *args, void *stream);

/* --------------------------------------------------------------------------
 * arc_attn_bwd: gradients of arc_attn_fwd (dense / GQA, causal or not, sinks).
 *
 * Source: "TransformerEngine: FA4 in context-parallel attention", flowchart:
 * the backward of each chunk is FA4's raw backward, from the saved O and LSE;
 * "pith-train: FA4 b19 return arity and MLA q/k concat" trains through the same
 * kernel.  The pages give no formula, so the gradients are the derivative of
 * the forward definition above (sink included):
 *     P = exp(scale q.k_j - LSE),  D_i = sum_d dO_id O_id,  delta_i = D_i - dLSE_i
 *     dV = P^T dO,   dS = P * (dO V^T - delta),   dQ = scale dS K,   dK = scale dS^T Q
 *     d sink_h = -sum_i exp(sink_h - LSE_i) delta_i
 * summed over the g query heads of each kv head for dK and dV.
 *
 *   q, k, v, o, lse   as the forward's arguments and outputs (o, lse: the
 *                     forward's results for these q, k, v, sinks)
 *   dout [B,H,Tq,Dv]  bf16, device, strides do_strides: the gradient of the loss wrt o
 *   dlse [B,H,Tq]     fp32, device, contiguous, or NULL: the gradient wrt lse
 *   dq [B,H,Tq,D], dk [B,Hkv,Tk,D], dv [B,Hkv,Tk,Dv]  bf16, device, written
 *   dsinks [H]        fp32, device, written when sinks != NULL
 * bf16 only, (D, Dv) in {(64,64), (128,128), (192,128)}; the tensor-core
 * layout needs each (b, kv) group's g*Tq query rows evenly spaced (head stride
 * == Tq * token stride) for q and dout, and 16-byte aligned rows and base
 * pointers everywhere.  P and dS are rounded to bf16 for the tensor cores, as in
 * the forward; accumulation is fp32.  Every sum runs in a fixed order (no
 * atomics): the same call twice gives the same bits.
 *   workspace  device, at least arc_attn_bwd_workspace_size(args) bytes, 256-byte
 *              aligned, overwritten; holds delta and, when the dK/dV work of a
 *              key tile is split over CTAs along the query rows, their fp32
 *              partials.  Its contents need no initialisation.
 * Launches: delta (and the sink gradient), dK/dV, the split reduction when
 * there is one, dQ.  Errors, before any launch: as arc_attn_fwd for shapes,
 * strides and pointers (ARC_ERR_UNSUPPORTED for another head-dim pair or
 * layout); a missing, short or unaligned workspace is ARC_ERR_WORKSPACE.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t B, H, Hkv, Tq, Tk, D, Dv;
    const void *q;    int64_t q_strides[3];
    const void *k;    int64_t k_strides[3];
    const void *v;    int64_t v_strides[3];
    const void *o;    int64_t o_strides[3];
    const void *dout; int64_t do_strides[3];
    const float *lse;
    const float *dlse;
    const float *sinks;
    void *dq;         int64_t dq_strides[3];
    void *dk;         int64_t dk_strides[3];
    void *dv;         int64_t dv_strides[3];
    float *dsinks;
    float scale;
    int32_t causal;
    uint32_t flags;
    uint32_t *status;
} arc_attn_bwd_args;

size_t arc_attn_bwd_workspace_size(const arc_attn_bwd_args *args);

arc_status arc_attn_bwd(const arc_attn_bwd_args *args, void *workspace, size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * arc_mla_bwd: gradients of arc_mla_fwd.
 *
 * Source: "pith-train: FA4 b19 return arity and MLA q/k concat", MLA section:
 * the model concatenates q = q_nope||q_rope and k = k_nope||k_rope and trains
 * through the attention call, so the gradients reach each part through that
 * concatenation.  They are those of arc_attn_bwd on the concatenated head dims
 * (d_qk = Dn + Dr, one kv head per query head, no sinks), split back:
 *     dq_nope, dq_rope   the first Dn and the last Dr columns of dQ
 *     dk_nope            the first Dn columns of each head's dK
 *     dk_rope            the sum over all H heads of the last Dr columns of dK
 *                        (k_rope is one tensor shared by every head)
 *     dv                 as arc_attn_bwd
 *
 *   q_nope ... v, o, lse   as arc_mla_fwd's arguments and outputs
 *   dout [B,H,Tq,Dv] bf16; dlse [B,H,Tq] fp32 or NULL
 *   dq_nope [B,H,Tq,Dn], dq_rope [B,H,Tq,Dr], dk_nope [B,H,Tk,Dn], dk_rope [B,Tk,Dr],
 *   dv [B,H,Tk,Dv]        bf16, device, written
 * (Dn + Dr, Dv) in {(128,128), (192,128)} with Dn, Dr multiples of 64; layout rules
 * as arc_attn_bwd.  workspace: at least arc_mla_bwd_workspace_size(args) bytes,
 * 256-byte aligned (delta, and each head's fp32 share of dk_rope before the
 * sum over heads, which runs in a fixed order).  Errors as arc_attn_bwd.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t B, H, Tq, Tk, Dn, Dr, Dv;
    const void *q_nope; int64_t q_nope_strides[3];
    const void *q_rope; int64_t q_rope_strides[3];
    const void *k_nope; int64_t k_nope_strides[3];
    const void *k_rope; int64_t k_rope_strides[2];
    const void *v;      int64_t v_strides[3];
    const void *o;      int64_t o_strides[3];
    const void *dout;   int64_t do_strides[3];
    const float *lse;
    const float *dlse;
    void *dq_nope;      int64_t dq_nope_strides[3];
    void *dq_rope;      int64_t dq_rope_strides[3];
    void *dk_nope;      int64_t dk_nope_strides[3];
    void *dk_rope;      int64_t dk_rope_strides[2];
    void *dv;           int64_t dv_strides[3];
    float scale;
    int32_t causal;
    uint32_t flags;
    uint32_t *status;
} arc_mla_bwd_args;

size_t arc_mla_bwd_workspace_size(const arc_mla_bwd_args *args);

arc_status arc_mla_bwd(const arc_mla_bwd_args *args, void *workspace, size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * Engagement record and helpers.
 *
 * arc_plan() answers, without launching anything, which kernel a call with
 * these arguments launches and with what tiling -- the per-call engagement
 * record ("ArcFlash ... rung 0", section D18: engagement is asserted, not
 * inferred from correct numbers; "unsloth llama.cpp ...", review note that
 * numerical equivalence is no proof the fast path ran).  It runs the same
 * host planner as the launch itself.  `op` is an arc_op and `args` points to
 * the matching args struct.
 * ------------------------------------------------------------------------ */
typedef struct {
    char kernel[64];      /* name of the kernel the call launches */
    int32_t tensor_cores; /* 1 if the hot loop runs on tcgen05 / mma tensor cores */
    int32_t tile_m;       /* query rows per CTA tile */
    int32_t tile_n;       /* keys per KV tile */
    int32_t d_slice;      /* d_v columns one CTA accumulates */
    int32_t n_ctas;       /* CTAs of the main launch */
    int32_t splits;       /* decode: KV splits per (sequence, kv head) */
    int32_t smem_bytes;   /* dynamic shared memory per CTA */
    int32_t tmem_cols;    /* TMEM columns allocated per CTA (0 if none) */
    int32_t launches;     /* kernels launched per call */
} arc_plan_info;

arc_status arc_plan(int32_t op, const void *args, arc_plan_info *out);

int32_t arc_abi_version(void);

const char *arc_status_string(arc_status s);

/* Synchronise `stream`, then read the device status word: ARC_OK if it is 0,
 * ARC_ERR_DEVICE_TIMEOUT otherwise (the word is left as it is). */
arc_status arc_check_device_error(const uint32_t *status, void *stream);

/* Launch one tiny kernel whose only wait is on a barrier nothing ever
 * arrives at, bounded by `timeout_ns`; it must report a timeout through
 * *status.  Exercises the same bounded-wait code the attention kernels use. */
arc_status arc_selftest_timeout(uint32_t *status, uint64_t timeout_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ARC_ATTN_H */
