/*
 * arc_oracle.c -- fp64 CPU oracle for exact softmax attention (forward).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file's library; the CUDA library
 * neither links nor calls it, and the two share no code.
 *
 * What it computes is the plain definition of exact scaled-dot-product
 * attention, one output row at a time, in double precision:
 *
 *   s_j   = scale * <q, k_j>                      for every visible key j
 *   m     = max(max_j s_j, sigma)                 sigma = per-head sink logit, or -inf
 *   l     = sum_j exp(s_j - m) + exp(sigma - m)
 *   O     = sum_j exp(s_j - m) v_j / l
 *   LSE   = m + ln(l)
 *
 * Sources: the forward output and per-row log-sum-exp are the two outputs of
 * the FA4 forward named in "pith-train PR: FA4 b19 return arity" (summary);
 * the sink as a per-head constant in each row's softmax denominator, the
 * kv-major GQA head map h = kv*g + rep, and exactness of query-row tiling are
 * from "ArcFlash - Arc's own attention kernel, rung 0" (sections "What rung 0
 * does" and "Mutations"); sparse top-k index lists from "TensorRT-LLM:
 * FlashMLA without -rdc" (timing paragraph); q8_0/q4_0 K/V blocks of 32
 * values plus an fp16 scale from "unsloth llama.cpp: dequantize q4_0/q8_0
 * K/V tiles in the FA MMA kernel" (summary paragraph).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - LSE is the natural log of the denominator of the *scaled* scores and
 *     includes the sink term; the sink logit is not multiplied by scale.
 *   - No visible key and no sink: O = 0 and LSE = -inf.
 *   - Causal alignment is bottom-right: query i sees keys j <= i + (Tk - Tq).
 *   - Sparse: an index outside [0, Skv) (e.g. -1) is masked; duplicates count
 *     once per slot; no causal mask is applied on top of the index list.
 *   - q8_0 value = d*q; q4_0 value = d*(n-8), element j in the low nibble of
 *     byte j and element j+16 in its high nibble; d is the block's fp16 scale.
 *
 * Mutation switch: oracle_set_mutation() plants one known mistake, so the
 * tests can show that their pins catch it (the pages' "four mutations, four
 * caught" discipline).  0 leaves the oracle correct.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum {
    MUT_NONE = 0,
    MUT_REP_MAJOR = 1,        /* GQA heads treated rep-major instead of kv-major */
    MUT_TILE_LOCAL_MASK = 2,  /* tiled mode: causal mask uses the tile-local row index */
    MUT_DROP_SINK = 3,        /* sink left out of the softmax denominator */
    MUT_TOP_LEFT_CAUSAL = 4,  /* causal mask aligned top-left instead of bottom-right */
    MUT_SWAP_NIBBLES = 5,     /* q4_0: low/high nibble roles swapped */
    MUT_MERGE_UNWEIGHTED = 6, /* merge: plain mean of the parts, no log-sum-exp weights */
    MUT_BWD_DROP_DELTA = 7,   /* read by the numpy backward (backward.py): D_i dropped from dS */
};

static int g_mutation = MUT_NONE;

void oracle_set_mutation(int m) { g_mutation = m; }
int oracle_get_mutation(void) { return g_mutation; }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* kv head read by query head h when H query heads share Hkv kv heads. */
static int kv_head_of(int h, int H, int Hkv)
{
    int g = H / Hkv;
    if (g_mutation == MUT_REP_MAJOR) return h % Hkv;
    return h / g;
}

/* Last visible key (inclusive) for query position i under a causal mask. */
static long causal_limit(long i, long Tq, long Tk)
{
    if (g_mutation == MUT_TOP_LEFT_CAUSAL) return i;
    return i + (Tk - Tq);
}

static double dot(const double *a, const double *b, int n)
{
    double s = 0.0;
    for (int d = 0; d < n; ++d) s += a[d] * b[d];
    return s;
}

/*
 * The softmax-weighted row.  s[0..n) are the scores of the visible keys in
 * key order, vrow[j] the matching value rows.  has_sink/sink give sigma.
 */
static void softmax_row(int n, const double *s, const double *const *vrow, int Dv,
                        int has_sink, double sink, double *o, double *lse)
{
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > m) m = s[j];
    if (has_sink && sink > m) m = sink;
    for (int d = 0; d < Dv; ++d) o[d] = 0.0;
    if (m == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j) l += exp(s[j] - m);
    if (has_sink && g_mutation != MUT_DROP_SINK) l += exp(sink - m);
    for (int j = 0; j < n; ++j) {
        double w = exp(s[j] - m);
        const double *vj = vrow[j];
        for (int d = 0; d < Dv; ++d) o[d] += w * vj[d];
    }
    for (int d = 0; d < Dv; ++d) o[d] /= l;
    *lse = m + log(l);
}

/*
 * Dense / GQA / MQA attention.
 *   q    [B,H,nr,Dqk]   the nr query rows to evaluate, at positions pos[nr] in [0,Tq)
 *   k    [B,Hkv,Tk,Dqk]
 *   v    [B,Hkv,Tk,Dv]
 *   sinks [H] or NULL
 *   o    [B,H,nr,Dv], lse [B,H,nr]
 * Returns 0, or -1 on bad arguments.
 */
int oracle_attn(int B, int H, int Hkv, int Tq, int Tk, int Dqk, int Dv, int nr, const int *pos,
                const double *q, const double *k, const double *v, double scale, int causal,
                const double *sinks, double *o, double *lse)
{
    if (B < 0 || H <= 0 || Hkv <= 0 || H % Hkv || Tq < 0 || Tk < 0 || nr < 0) return -1;
    long rows = (long)B * H * nr;
    int fail = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Tk > 0 ? Tk : 1));
        const double **vr = (const double **)malloc(sizeof(double *) * (Tk > 0 ? Tk : 1));
        if (!s || !vr) fail = 1;
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < rows; ++r) {
            if (!s || !vr) continue;
            long b = r / ((long)H * nr), h = (r / nr) % H, ii = r % nr;
            long kv = kv_head_of((int)h, H, Hkv);
            const double *qr = q + r * Dqk;
            long last = causal ? causal_limit(pos[ii], Tq, Tk) : (long)Tk - 1;
            if (last > Tk - 1) last = Tk - 1;
            int n = 0;
            for (long j = 0; j <= last; ++j) {
                const double *kj = k + (((long)b * Hkv + kv) * Tk + j) * Dqk;
                s[n] = scale * dot(qr, kj, Dqk);
                vr[n] = v + (((long)b * Hkv + kv) * Tk + j) * Dv;
                ++n;
            }
            softmax_row(n, s, vr, Dv, sinks != NULL, sinks ? sinks[h] : 0.0, o + r * Dv, lse + r);
        }
        free(s);
        free((void *)vr);
    }
    return fail ? -1 : 0;
}

/*
 * The same attention evaluated through query-row tiles: rows of every head are
 * processed in tiles of R rows, R the largest count whose fp32 score block
 * H*R*Tk*4 bytes fits tile_bytes (at least 1).  Each tile's score block is
 * formed in full and then masked with the rows' absolute positions.
 * q [B,H,Tq,Dqk]; outputs as oracle_attn with nr = Tq.  *n_tiles gets the
 * number of tiles per batch element.
 */
int oracle_attn_tiled(int B, int H, int Hkv, int Tq, int Tk, int Dqk, int Dv,
                      const double *q, const double *k, const double *v, double scale, int causal,
                      const double *sinks, long long tile_bytes, double *o, double *lse, int *n_tiles)
{
    if (B < 0 || H <= 0 || Hkv <= 0 || H % Hkv || Tq <= 0 || Tk <= 0) return -1;
    long long per_row = (long long)H * Tk * 4;
    long R = (long)(tile_bytes / per_row);
    if (R < 1) R = 1;
    if (R > Tq) R = Tq;
    long nt = (Tq + R - 1) / R;
    if (n_tiles) *n_tiles = (int)nt;
    double *S = (double *)malloc(sizeof(double) * (size_t)H * R * Tk);
    unsigned char *vis = (unsigned char *)malloc((size_t)R * Tk);
    if (!S || !vis) {
        free(S);
        free(vis);
        return -1;
    }
    for (long b = 0; b < B; ++b) {
        for (long t0 = 0; t0 < Tq; t0 += R) {
            long rows = (Tq - t0 < R) ? Tq - t0 : R;
            /* visibility of (row, key) for this tile */
            for (long i = 0; i < rows; ++i) {
                long p = (g_mutation == MUT_TILE_LOCAL_MASK) ? i : t0 + i;
                long last = causal ? causal_limit(p, Tq, Tk) : (long)Tk - 1;
                for (long j = 0; j < Tk; ++j) vis[i * Tk + j] = (j <= last);
            }
#pragma omp parallel for schedule(static)
            for (long hi = 0; hi < (long)H * rows; ++hi) {
                long h = hi / rows, i = hi % rows;
                long kv = kv_head_of((int)h, H, Hkv);
                const double *qr = q + (((long)b * H + h) * Tq + t0 + i) * Dqk;
                double *Srow = S + ((long)h * R + i) * Tk;
                for (long j = 0; j < Tk; ++j)
                    Srow[j] = scale * dot(qr, k + (((long)b * Hkv + kv) * Tk + j) * Dqk, Dqk);
            }
#pragma omp parallel
            {
                double *s = (double *)malloc(sizeof(double) * Tk);
                const double **vr = (const double **)malloc(sizeof(double *) * Tk);
#pragma omp for schedule(static)
                for (long hi = 0; hi < (long)H * rows; ++hi) {
                    long h = hi / rows, i = hi % rows;
                    long kv = kv_head_of((int)h, H, Hkv);
                    const double *Srow = S + ((long)h * R + i) * Tk;
                    int n = 0;
                    for (long j = 0; j < Tk; ++j) {
                        if (!vis[i * Tk + j]) continue;
                        s[n] = Srow[j];
                        vr[n] = v + (((long)b * Hkv + kv) * Tk + j) * Dv;
                        ++n;
                    }
                    long r = ((long)b * H + h) * Tq + t0 + i;
                    softmax_row(n, s, vr, Dv, sinks != NULL, sinks ? sinks[h] : 0.0, o + r * Dv,
                                lse + r);
                }
                free(s);
                free((void *)vr);
            }
        }
    }
    free(S);
    free(vis);
    return 0;
}

/*
 * The GQA fold: per (b, kv) the g*Tq query rows are one row block,
 * fold row r <-> (rep = r / Tq, t = r mod Tq), query head h = kv*g + rep.
 * q [B,H,Tq,Dqk]; o_fold [B,Hkv,g*Tq,Dv]; lse_fold [B,Hkv,g*Tq].
 * With q contiguous, o_fold has the memory layout of o [B,H,Tq,Dv].
 */
int oracle_attn_fold(int B, int H, int Hkv, int Tq, int Tk, int Dqk, int Dv,
                     const double *q, const double *k, const double *v, double scale, int causal,
                     const double *sinks, double *o_fold, double *lse_fold)
{
    if (B < 0 || H <= 0 || Hkv <= 0 || H % Hkv || Tq <= 0 || Tk < 0) return -1;
    long g = H / Hkv;
    long rows = (long)B * Hkv * g * Tq;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Tk > 0 ? Tk : 1));
        const double **vr = (const double **)malloc(sizeof(double *) * (Tk > 0 ? Tk : 1));
#pragma omp for schedule(dynamic, 4)
        for (long x = 0; x < rows; ++x) {
            long b = x / (Hkv * g * Tq), kv = (x / (g * Tq)) % Hkv, r = x % (g * Tq);
            long rep = r / Tq, t = r % Tq;
            long h = (g_mutation == MUT_REP_MAJOR) ? rep * Hkv + kv : kv * g + rep;
            const double *qr = q + (((long)b * H + h) * Tq + t) * Dqk;
            long last = causal ? causal_limit(t, Tq, Tk) : (long)Tk - 1;
            if (last > Tk - 1) last = Tk - 1;
            int n = 0;
            for (long j = 0; j <= last; ++j) {
                s[n] = scale * dot(qr, k + (((long)b * Hkv + kv) * Tk + j) * Dqk, Dqk);
                vr[n] = v + (((long)b * Hkv + kv) * Tk + j) * Dv;
                ++n;
            }
            softmax_row(n, s, vr, Dv, sinks != NULL, sinks ? sinks[h] : 0.0, o_fold + x * Dv,
                        lse_fold + x);
        }
        free(s);
        free((void *)vr);
    }
    return 0;
}

/*
 * MLA attention with asymmetric head dims: q = q_nope || q_rope and
 * k = k_nope[h] || k_rope, where k_rope is one tensor shared by all heads.
 *   q_nope [B,H,nr,Dn], q_rope [B,H,nr,Dr] (rows at positions pos[nr])
 *   k_nope [B,H,Tk,Dn], k_rope [B,Tk,Dr], v [B,H,Tk,Dv]
 *   o [B,H,nr,Dv], lse [B,H,nr]
 */
int oracle_mla(int B, int H, int Tq, int Tk, int Dn, int Dr, int Dv, int nr, const int *pos,
               const double *q_nope, const double *q_rope, const double *k_nope,
               const double *k_rope, const double *v, double scale, int causal, double *o,
               double *lse)
{
    if (B < 0 || H <= 0 || Tq < 0 || Tk < 0 || nr < 0) return -1;
    long rows = (long)B * H * nr;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Tk > 0 ? Tk : 1));
        const double **vr = (const double **)malloc(sizeof(double *) * (Tk > 0 ? Tk : 1));
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < rows; ++r) {
            long b = r / ((long)H * nr), h = (r / nr) % H, ii = r % nr;
            const double *qn = q_nope + r * Dn, *qr = q_rope + r * Dr;
            long last = causal ? causal_limit(pos[ii], Tq, Tk) : (long)Tk - 1;
            if (last > Tk - 1) last = Tk - 1;
            int n = 0;
            for (long j = 0; j <= last; ++j) {
                const double *kn = k_nope + (((long)b * H + h) * Tk + j) * Dn;
                const double *kr = k_rope + ((long)b * Tk + j) * Dr;
                s[n] = scale * (dot(qn, kn, Dn) + dot(qr, kr, Dr));
                vr[n] = v + (((long)b * H + h) * Tk + j) * Dv;
                ++n;
            }
            softmax_row(n, s, vr, Dv, 0, 0.0, o + r * Dv, lse + r);
        }
        free(s);
        free((void *)vr);
    }
    return 0;
}

/*
 * Sparse attention over per-query index lists into a pool shared by all heads.
 *   q [nq,H,Dqk], kv [Skv,Dqk], v [Skv,Dv] or NULL (then V row = kv row[0..Dv))
 *   idx [nq,topk] int32; a slot outside [0,Skv) is masked
 *   sinks [H] or NULL; o [nq,H,Dv], lse [nq,H]
 */
int oracle_sparse(int nq, int H, int Skv, int Dqk, int Dv, int topk, const double *q,
                  const double *kv, const double *v, const int32_t *idx, double scale,
                  const double *sinks, double *o, double *lse)
{
    if (nq < 0 || H <= 0 || Skv < 0 || topk < 0) return -1;
    if (!v && Dv > Dqk) return -1;
    long rows = (long)nq * H;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (topk > 0 ? topk : 1));
        const double **vr = (const double **)malloc(sizeof(double *) * (topk > 0 ? topk : 1));
#pragma omp for schedule(dynamic, 8)
        for (long r = 0; r < rows; ++r) {
            long i = r / H, h = r % H;
            const double *qr = q + r * Dqk;
            int n = 0;
            for (long slot = 0; slot < topk; ++slot) {
                long j = idx[i * (long)topk + slot];
                if (j < 0 || j >= Skv) continue;
                s[n] = scale * dot(qr, kv + j * (long)Dqk, Dqk);
                vr[n] = v ? v + j * (long)Dv : kv + j * (long)Dqk;
                ++n;
            }
            softmax_row(n, s, vr, Dv, sinks != NULL, sinks ? sinks[h] : 0.0, o + r * Dv, lse + r);
        }
        free(s);
        free((void *)vr);
    }
    return 0;
}

/* IEEE-754 binary16 -> double, from the format's definition. */
static double half_to_double(uint16_t x)
{
    int sign = (x >> 15) & 1, e = (x >> 10) & 31, f = x & 1023;
    double val;
    if (e == 0)
        val = ldexp((double)f, -24);
    else if (e == 31)
        val = f ? NAN : INFINITY;
    else
        val = ldexp(1.0 + f / 1024.0, e - 15);
    return sign ? -val : val;
}

#define KV_Q8_0 8
#define KV_Q4_0 2

/* Dequantise one head row of D values (D/32 blocks) into out[D]. */
static int dequant_row(int kv_type, const uint8_t *row, int D, double *out)
{
    int nb = D / 32;
    for (int bi = 0; bi < nb; ++bi) {
        if (kv_type == KV_Q8_0) {
            const uint8_t *blk = row + bi * 34;
            double d = half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
            for (int j = 0; j < 32; ++j) out[bi * 32 + j] = d * (double)(int8_t)blk[2 + j];
        } else if (kv_type == KV_Q4_0) {
            const uint8_t *blk = row + bi * 18;
            double d = half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
            for (int j = 0; j < 16; ++j) {
                int lo = blk[2 + j] & 15, hi = blk[2 + j] >> 4;
                if (g_mutation == MUT_SWAP_NIBBLES) {
                    int t = lo;
                    lo = hi;
                    hi = t;
                }
                out[bi * 32 + j] = d * (double)(lo - 8);
                out[bi * 32 + j + 16] = d * (double)(hi - 8);
            }
        } else {
            return -1;
        }
    }
    return 0;
}

/* Dequantise a whole cache [n_cells,Hkv,D/32 blocks] into out [n_cells,Hkv,D]. */
int oracle_dequant_cache(int kv_type, int n_cells, int Hkv, int D, const uint8_t *cache,
                         double *out)
{
    int bb = kv_type == KV_Q8_0 ? 34 : (kv_type == KV_Q4_0 ? 18 : 0);
    if (!bb || D % 32) return -1;
    long rowb = (long)(D / 32) * bb;
    for (long r = 0; r < (long)n_cells * Hkv; ++r)
        if (dequant_row(kv_type, cache + r * rowb, D, out + r * D)) return -1;
    return 0;
}

/*
 * Multi-sequence decode over one unified quantised cache.
 *   q [n_tok,H,D] (double), caches [n_cells,Hkv,D/32 blocks] (bytes)
 *   sequence s: tokens q_begin[s]..+n_q[s], cells kv_begin[s]..+n_kv[s];
 *   its token t (0-based within the sequence) sees cells
 *   kv_begin[s] .. kv_begin[s] + n_kv[s] - n_q[s] + t.
 *   o [n_tok,H,D], lse [n_tok,H]
 */
int oracle_decode_q(int kv_type, int n_seq, const int32_t *q_begin, const int32_t *n_q,
                    const int32_t *kv_begin, const int32_t *n_kv, int n_tok, int H, int Hkv,
                    int D, const double *q, int n_cells, const uint8_t *k_cache,
                    const uint8_t *v_cache, double scale, double *o, double *lse)
{
    int bb = kv_type == KV_Q8_0 ? 34 : (kv_type == KV_Q4_0 ? 18 : 0);
    if (!bb || D % 32 || H % Hkv) return -1;
    long rowb = (long)(D / 32) * bb;
    long maxkv = 1;
    for (int s = 0; s < n_seq; ++s) {
        if (n_kv[s] < n_q[s] || kv_begin[s] < 0 || kv_begin[s] + n_kv[s] > n_cells) return -1;
        if (q_begin[s] < 0 || q_begin[s] + n_q[s] > n_tok) return -1;
        if (n_kv[s] > maxkv) maxkv = n_kv[s];
    }
    int fail = 0;
    for (int s = 0; s < n_seq; ++s) {
        long nk = n_kv[s];
        /* dequantised K/V of this sequence, per kv head: [Hkv][nk][D] */
        double *Kd = (double *)malloc(sizeof(double) * (size_t)Hkv * (nk ? nk : 1) * D);
        double *Vd = (double *)malloc(sizeof(double) * (size_t)Hkv * (nk ? nk : 1) * D);
        if (!Kd || !Vd) {
            free(Kd);
            free(Vd);
            return -1;
        }
        for (long c = 0; c < nk; ++c)
            for (int kh = 0; kh < Hkv; ++kh) {
                long cell = kv_begin[s] + c;
                if (dequant_row(kv_type, k_cache + (cell * Hkv + kh) * rowb, D,
                                Kd + ((long)kh * nk + c) * D) ||
                    dequant_row(kv_type, v_cache + (cell * Hkv + kh) * rowb, D,
                                Vd + ((long)kh * nk + c) * D))
                    fail = 1;
            }
        long rows = (long)n_q[s] * H;
#pragma omp parallel
        {
            double *sc = (double *)malloc(sizeof(double) * maxkv);
            const double **vr = (const double **)malloc(sizeof(double *) * maxkv);
#pragma omp for schedule(static)
            for (long x = 0; x < rows; ++x) {
                long t = x / H, h = x % H;
                long kh = kv_head_of((int)h, H, Hkv);
                long tok = q_begin[s] + t;
                const double *qr = q + (tok * H + h) * D;
                long last = nk - n_q[s] + t;
                int n = 0;
                for (long c = 0; c <= last; ++c) {
                    sc[n] = scale * dot(qr, Kd + (kh * nk + c) * D, D);
                    vr[n] = Vd + (kh * nk + c) * D;
                    ++n;
                }
                softmax_row(n, sc, vr, D, 0, 0.0, o + (tok * H + h) * D, lse + tok * H + h);
            }
            free(sc);
            free((void *)vr);
        }
        free(Kd);
        free(Vd);
    }
    return fail ? -1 : 0;
}

/*
 * Merge of results over disjoint key sets ("TransformerEngine: FA4 in
 * context-parallel attention", flowchart): when the keys of a row are split
 * over parts and part i gives a normalised output O_i and log-sum-exp LSE_i
 * over its own keys, then over all the keys
 *
 *   LSE = ln( sum_i exp(LSE_i) + exp(sigma) )      sigma = sink logit, or -inf
 *   O   = sum_i exp(LSE_i - LSE) O_i
 *
 * (the sink enters once, here).  A part with LSE_i = -inf is empty.  A row
 * with every part empty and no sink gets O = 0 and LSE = -inf.  The largest
 * term is factored out of the sum only to keep exp finite.
 *
 * o_parts [n_parts][rows][dv], lse_parts [n_parts][rows], sink_row [rows] or NULL.
 */
int oracle_merge(int n_parts, long rows, int dv, const double *o_parts, const double *lse_parts,
                 const double *sink_row, double *o, double *lse)
{
    if (n_parts < 1 || rows < 0 || dv < 1) return -1;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        const double sigma = sink_row ? sink_row[r] : -INFINITY;
        double mx = sigma;
        for (int i = 0; i < n_parts; ++i) mx = fmax(mx, lse_parts[(long)i * rows + r]);
        double *orow = o + r * dv;
        for (int d = 0; d < dv; ++d) orow[d] = 0.0;
        if (mx == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = (sigma == -INFINITY) ? 0.0 : exp(sigma - mx);
        for (int i = 0; i < n_parts; ++i) {
            const double li = lse_parts[(long)i * rows + r];
            if (li != -INFINITY) sum += exp(li - mx);
        }
        const double L = mx + log(sum);
        lse[r] = L;
        for (int i = 0; i < n_parts; ++i) {
            const double li = lse_parts[(long)i * rows + r];
            if (li == -INFINITY) continue;
            const double w = (g_mutation == MUT_MERGE_UNWEIGHTED) ? 1.0 / n_parts : exp(li - L);
            const double *pr = o_parts + ((long)i * rows + r) * dv;
            for (int d = 0; d < dv; ++d) orow[d] += w * pr[d];
        }
    }
    return 0;
}
