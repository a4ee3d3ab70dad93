/*
 * oracle.c -- plain FP64 CPU reference of the W4A16 quantized-expert MoE layer.
 *
 * TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * constant with the CUDA path; it is slow and written to be checked by eye.
 *
 * What it computes, and where each step comes from:
 *
 *  - W4A16: 4-bit integer weights, fp16 activations.
 *      "GLM-5.3-Flash 320B MoEを4枚のCMP 170HXで動かすvLLMレシピ" (648news),
 *      section "OpenAI互換APIで動く320BパラメータのMoE構成".
 *  - int4 codes with one scale per output row (symmetric, no zero point).
 *      "Show HN: 低速のコンピュータでGLM 5.2を動かす方法" (hakusoku), section
 *      "実装済み機能", the int8/int4/int2 kernels with per-row scales.
 *  - NVFP4 (E2M1 codes, one E4M3 scale per 16 elements, fp32 tensor scale) decoded
 *    inside the matmul.  "GTX 1070向け35BパラメータMoEモデル推論エンジン公開"
 *    (648news), section "VRAMとシステムメモリで重みを分割する設計" and the NVFP4
 *    entry of "用語の注釈"; the bit layouts are those of the OCP Microscaling
 *    Formats specification v1.0 (E2M1, E4M3 "FN").
 *  - DeepSeek-V3-style sigmoid router with a shared expert.  hakusoku page,
 *    section "実装済み機能".  The router formula is the DeepSeek-V3 one: sigmoid
 *    scores, a per-expert bias that only affects selection, top-k, combine weights
 *    = scores of the chosen experts normalised to sum 1 and multiplied by the
 *    routed scaling factor.  No group-limited routing (one group).
 *  - Batch MoE union: every unique expert of a batch is read once and applied to
 *    all positions routed to it.  hakusoku page, section "実装済み機能".
 *  - Deterministic MoE block order.  648news GLM-5.3 page, section
 *    "Ampere世代のGPU向けに最適化された独自カーネル群".
 *
 * Readings taken where the pages are silent (each also listed in the design notes):
 *  - nibble order: element 2b in the low nibble of byte b, 2b+1 in the high nibble;
 *    int4 codes are two's complement (0x8..0xF -> -8..-1).
 *  - NVFP4 blocks of 16 run along K of each output row, same nibble order.
 *  - router logits are accumulated in fp64 and rounded to fp32; sigmoid in fp64
 *    rounded to fp32; selection score = fp32 add of score and bias; top-k ties go
 *    to the lower expert index; combine weight w = scaling * (s_j / sum_j s_j) in
 *    fp64, stored as fp32.
 *  - grouping: counts, exclusive offsets, permutation of assignment ids
 *    a = t*k + j ordered by expert, ascending a inside an expert.
 *  - expert FFN: g = W_g x, u = W_u x, h = SiLU(g) * u, y_e = W_d h, all fp64,
 *    sums in ascending index order.
 *  - combine: y_t = shared(x_t) + sum_{j=0..k-1} w_tj * y_{e_tj}(x_t), the shared
 *    expert with weight 1.
 *  - int8 and int2 codes with one scale per output row (hakusoku page, section
 *    "実装済み機能": int8/int4/int2 kernels with per-row scales).  Readings: int8 is one
 *    two's-complement byte per weight; int2 packs four two's-complement codes in
 *    [-2, 1] per byte, element 4b+i in bits 2i..2i+1 (the int4 order continued).
 *  - per-row quantisation (hakusoku page, section "実装済み機能": the offline FP8 -> int4
 *    conversion tool).  Reading: symmetric, scale = max|w| / (2^(bits-1) - 1) rounded
 *    to fp32, code = round-half-even(w / scale) with that fp32 scale, clamped to the
 *    code range; an all-zero row gets scale 0 and zero codes.
 *  - adaptive expert top-p (hakusoku page, section "実行・チューニングパラメータ":
 *    the --topp option, which names the idea and its effect but not the rule).
 *    Reading: after top-k, order the k chosen experts by their score s (descending,
 *    equal scores -> lower expert index) and keep the shortest leading run whose
 *    score sum reaches top_p times the sum over all k (at least one expert): expert
 *    r of that order is kept iff the sum of the r before it is below top_p * S, all
 *    sums in fp64 in the stated order, S summed in top-k order.  Kept experts keep
 *    their top-k order and move to the front; their weights are scaling * s / S'
 *    (S' the kept scores summed in top-k order); the rest are index -1, weight 0,
 *    and take no part in grouping or combine.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ------------------------------------------------------------ scalar decodes */

double orc_half_to_double(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);            /* (1 + m/1024) * 2^(e-15) */
    return s ? -v : v;
}

int orc_int4_at(const uint8_t *row, long k)
{
    unsigned b = row[k >> 1];
    int n = (k & 1) ? (int)(b >> 4) : (int)(b & 15);
    return n >= 8 ? n - 16 : n;
}

int orc_int8_at(const uint8_t *row, long k)
{
    int n = row[k];
    return n >= 128 ? n - 256 : n;
}

int orc_int2_at(const uint8_t *row, long k)
{
    unsigned b = row[k >> 2];
    int n = (int)((b >> (2 * (k & 3))) & 3u);
    return n >= 2 ? n - 4 : n;
}

double orc_e2m1_to_double(unsigned code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);   /* bias 1 */
    return s ? -v : v;
}

double orc_e4m3_to_double(uint8_t b)
{
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9)                     /* m/8 * 2^-6 */
                        : ldexp(1.0 + m / 8.0, e - 7);             /* bias 7 */
    return s ? -v : v;
}

/* bytes of one row of K codes */
static size_t row_bytes(int format, long K)
{
    return format == ORC_INT8 ? (size_t)K : format == ORC_INT2 ? (size_t)(K / 4) : (size_t)(K / 2);
}

/* dequantised weight (row n, column k) of one matrix */
static double wq(const orc_matrix *M, long n, long k)
{
    const uint8_t *row = M->codes + (size_t)n * row_bytes(M->format, M->K);
    if (M->format == ORC_INT4) {
        return (double)orc_int4_at(row, k) * (double)M->row_scale[n];
    } else if (M->format == ORC_INT8) {
        return (double)orc_int8_at(row, k) * (double)M->row_scale[n];
    } else if (M->format == ORC_INT2) {
        return (double)orc_int2_at(row, k) * (double)M->row_scale[n];
    } else {
        unsigned b = row[k >> 1];
        unsigned c = (k & 1) ? (b >> 4) : (b & 15);
        uint8_t sb = M->block_scale[(size_t)n * (size_t)(M->K / 16) + (size_t)(k / 16)];
        return orc_e2m1_to_double(c) * orc_e4m3_to_double(sb) * (double)M->tensor_scale;
    }
}

/* all dequantised weights of one matrix, [N][K] */
void orc_dequant_matrix(const orc_matrix *M, double *out)
{
    for (long n = 0; n < M->N; n++)
        for (long k = 0; k < M->K; k++) out[(size_t)n * (size_t)M->K + (size_t)k] = wq(M, n, k);
}

/* ------------------------------------------------------------ quantisation */

void orc_quantize_rows(const float *w, int N, int K, int bits, uint8_t *codes, float *scale)
{
    int qmax = (1 << (bits - 1)) - 1, qmin = -(1 << (bits - 1));
    size_t rb = row_bytes(bits == 8 ? ORC_INT8 : bits == 2 ? ORC_INT2 : ORC_INT4, K);
    memset(codes, 0, rb * (size_t)N);
    for (int n = 0; n < N; n++) {
        double amax = 0.0;
        for (int k = 0; k < K; k++) {
            double a = fabs((double)w[(size_t)n * K + k]);
            if (a > amax) amax = a;
        }
        float sc = (float)(amax / qmax);
        scale[n] = sc;
        uint8_t *row = codes + (size_t)n * rb;
        for (int k = 0; k < K; k++) {
            int q = 0;
            if (sc > 0.0f) {
                double v = rint((double)w[(size_t)n * K + k] / (double)sc);   /* ties to even */
                if (v > qmax) v = qmax;
                if (v < qmin) v = qmin;
                q = (int)v;
            }
            unsigned u = (unsigned)q;
            if (bits == 8) row[k] = (uint8_t)(u & 255u);
            else if (bits == 4) row[k >> 1] |= (uint8_t)((u & 15u) << (4 * (k & 1)));
            else row[k >> 2] |= (uint8_t)((u & 3u) << (2 * (k & 3)));
        }
    }
}

/* ------------------------------------------------------------------ router */

void orc_router_logits(const uint16_t *x, int T, int H, const float *Wr, int E, float *logits)
{
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            double acc = 0.0;
            for (int h = 0; h < H; h++)
                acc += (double)Wr[(size_t)e * H + h] * orc_half_to_double(x[(size_t)t * H + h]);
            logits[(size_t)t * E + e] = (float)acc;
        }
}

float orc_sigmoid_f32(float logit)
{
    return (float)(1.0 / (1.0 + exp(-(double)logit)));
}

void orc_route(const float *logits, const float *bias, int T, int E, int k, double scaling,
               int32_t *topk_idx, float *topk_w, float *sel_out, float *gap_out)
{
    orc_route_p(logits, bias, T, E, k, scaling, 0.0, topk_idx, topk_w, sel_out, gap_out);
}

/* Adaptive top-p on one token's k chosen experts (see the header comment).  Rewrites
 * idx / w in place; returns the smallest distance of a cumulative share from top_p
 * (how close the decision came to flipping), or +inf when nothing was decided. */
static double top_p_token(const float *s, int k, double scaling, double top_p, int32_t *idx, float *w)
{
    double S = 0.0;
    for (int j = 0; j < k; j++) S += (double)s[idx[j]];
    /* order of the k experts by score: rank[j] = number of experts ahead of j */
    int *rank = (int *)malloc(sizeof(int) * (size_t)k);
    int *at = (int *)malloc(sizeof(int) * (size_t)k);
    for (int j = 0; j < k; j++) {
        int r = 0;
        for (int i = 0; i < k; i++) {
            float si = s[idx[i]], sj = s[idx[j]];
            if (si > sj || (si == sj && idx[i] < idx[j])) r++;
        }
        rank[j] = r;
        at[r] = j;
    }
    char *keep = (char *)calloc((size_t)k, 1);
    double before = 0.0, margin = INFINITY;
    for (int r = 0; r < k; r++) {                      /* walk the score order */
        if (r > 0) {
            double d = fabs(before / S - top_p);
            if (d < margin) margin = d;
        }
        keep[at[r]] = before < top_p * S;
        before += (double)s[idx[at[r]]];
    }
    double S2 = 0.0;
    for (int j = 0; j < k; j++)
        if (keep[j]) S2 += (double)s[idx[j]];
    int32_t *old = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    memcpy(old, idx, sizeof(int32_t) * (size_t)k);
    int m = 0;
    for (int j = 0; j < k; j++)
        if (keep[j]) {
            idx[m] = old[j];
            w[m] = (float)(scaling * ((double)s[old[j]] / S2));
            m++;
        }
    for (; m < k; m++) {
        idx[m] = -1;
        w[m] = 0.0f;
    }
    free(rank);
    free(at);
    free(keep);
    free(old);
    return margin;
}

void orc_route_p(const float *logits, const float *bias, int T, int E, int k, double scaling,
                 double top_p, int32_t *topk_idx, float *topk_w, float *sel_out, float *gap_out)
{
    float *s = (float *)malloc(sizeof(float) * (size_t)E);
    float *sel = (float *)malloc(sizeof(float) * (size_t)E);
    char *taken = (char *)malloc((size_t)E);
    for (int t = 0; t < T; t++) {
        for (int e = 0; e < E; e++) {
            s[e] = orc_sigmoid_f32(logits[(size_t)t * E + e]);
            sel[e] = s[e] + bias[e];                 /* one fp32 add */
            if (sel_out) sel_out[(size_t)t * E + e] = sel[e];
        }
        memset(taken, 0, (size_t)E);
        float last = 0.0f;
        for (int j = 0; j < k; j++) {                /* k passes of an argmax */
            int best = -1;
            for (int e = 0; e < E; e++)
                if (!taken[e] && (best < 0 || sel[e] > sel[best])) best = e;
            taken[best] = 1;
            topk_idx[(size_t)t * k + j] = best;
            last = sel[best];
        }
        double sum = 0.0;
        for (int j = 0; j < k; j++) sum += (double)s[topk_idx[(size_t)t * k + j]];
        for (int j = 0; j < k; j++)
            topk_w[(size_t)t * k + j] =
                (float)(scaling * ((double)s[topk_idx[(size_t)t * k + j]] / sum));
        float gap = INFINITY;
        if (k < E) {
            /* margin between the k-th chosen and the best unchosen selection score */
            float next = -INFINITY;
            for (int e = 0; e < E; e++)
                if (!taken[e] && sel[e] > next) next = sel[e];
            gap = (float)((double)last - (double)next);
        }
        if (top_p > 0.0 && top_p < 1.0) {
            /* the top-p decision's own margin joins the gap (both decide integers) */
            double m = top_p_token(s, k, scaling, top_p, topk_idx + (size_t)t * k, topk_w + (size_t)t * k);
            if (m < (double)gap) gap = (float)m;
        }
        if (gap_out) gap_out[t] = gap;
    }
    free(s);
    free(sel);
    free(taken);
}

/* ---------------------------------------------------------------- grouping */

void orc_group(const int32_t *topk_idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
               int32_t *perm, int32_t *unique, int32_t *n_unique)
{
    int n = T * k;
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int a = 0; a < n; a++)
        if (topk_idx[a] >= 0) counts[topk_idx[a]]++;   /* -1: dropped by top-p */
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    for (int a = 0; a < n; a++) {                      /* ascending a: stable */
        int e = topk_idx[a];
        if (e >= 0) perm[offsets[e] + fill[e]++] = a;
    }
    free(fill);
    int u = 0;
    for (int e = 0; e < E; e++)
        if (counts[e] > 0) unique[u++] = e;
    *n_unique = u;
}

/* -------------------------------------------------------------- expert FFN */

void orc_expert_ffn(const orc_matrix *Wg, const orc_matrix *Wu, const orc_matrix *Wd,
                    const double *x, double *h_out, double *y)
{
    int I = Wg->N, H = Wg->K;
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < I; n++) {
        double g = 0.0, u = 0.0;
        for (int kk = 0; kk < H; kk++) {
            g += wq(Wg, n, kk) * x[kk];
            u += wq(Wu, n, kk) * x[kk];
        }
        h[n] = g / (1.0 + exp(-g)) * u;               /* SiLU(g) * u */
    }
#pragma omp parallel for schedule(static)
    for (int m = 0; m < Wd->N; m++) {
        double acc = 0.0;
        for (int n = 0; n < I; n++) acc += wq(Wd, m, n) * h[n];
        y[m] = acc;
    }
    if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)I);
    free(h);
}

static orc_matrix routed_matrix(const orc_layer *L, int which, int e)
{
    orc_matrix M;
    memset(&M, 0, sizeof M);
    M.format = L->format;
    int rows = which == 2 ? L->H : L->I;
    int K = which == 2 ? L->I : L->H;
    M.N = rows;
    M.K = K;
    const uint8_t *codes = which == 0 ? L->g : which == 1 ? L->u : L->d;
    M.codes = codes + (size_t)e * (size_t)rows * row_bytes(L->format, K);
    if (L->format != ORC_NVFP4) {   /* row-scaled integer codes */
        const float *sc = which == 0 ? L->sg : which == 1 ? L->su : L->sd;
        M.row_scale = sc + (size_t)e * (size_t)rows;
    } else {
        const uint8_t *bs = which == 0 ? L->bg : which == 1 ? L->bu : L->bd;
        const float *ts = which == 0 ? L->tg : which == 1 ? L->tu : L->td;
        M.block_scale = bs + (size_t)e * (size_t)rows * (size_t)(K / 16);
        M.tensor_scale = ts[e];
    }
    return M;
}

static orc_matrix shared_matrix(const orc_layer *L, int which)
{
    orc_matrix M;
    memset(&M, 0, sizeof M);
    M.format = L->format;
    M.N = which == 2 ? L->H : L->I_sh;
    M.K = which == 2 ? L->I_sh : L->H;
    M.codes = which == 0 ? L->sh_g : which == 1 ? L->sh_u : L->sh_d;
    if (L->format != ORC_NVFP4) {   /* row-scaled integer codes */
        M.row_scale = which == 0 ? L->sh_sg : which == 1 ? L->sh_su : L->sh_sd;
    } else {
        M.block_scale = which == 0 ? L->sh_bg : which == 1 ? L->sh_bu : L->sh_bd;
        M.tensor_scale = which == 0 ? L->sh_tg : which == 1 ? L->sh_tu : L->sh_td;
    }
    return M;
}

void orc_routed_expert(const orc_layer *L, int e, const double *x, double *h_out, double *y)
{
    orc_matrix g = routed_matrix(L, 0, e), u = routed_matrix(L, 1, e), d = routed_matrix(L, 2, e);
    orc_expert_ffn(&g, &u, &d, x, h_out, y);
}

void orc_shared_expert(const orc_layer *L, const double *x, double *h_out, double *y)
{
    orc_matrix g = shared_matrix(L, 0), u = shared_matrix(L, 1), d = shared_matrix(L, 2);
    orc_expert_ffn(&g, &u, &d, x, h_out, y);
}

/* ------------------------------------------------------------------ drivers */

static void decode_tokens(const uint16_t *x, int T, int H, double *xd)
{
    for (size_t i = 0; i < (size_t)T * H; i++) xd[i] = orc_half_to_double(x[i]);
}

static void route_all(const orc_layer *L, const uint16_t *x, int T, const float *logits_in,
                      orc_result *R)
{
    if (logits_in)
        memcpy(R->logits, logits_in, sizeof(float) * (size_t)T * L->E);
    else
        orc_router_logits(x, T, L->H, L->Wr, L->E, R->logits);
    orc_route_p(R->logits, L->bias, T, L->E, L->k, L->scaling, L->top_p, R->topk_idx, R->topk_w,
                R->sel, R->gap);
}

static void combine(const orc_layer *L, int T, const double *y_assign, const double *y_shared,
                    const int32_t *topk_idx, const float *topk_w, double *y)
{
    int H = L->H, k = L->k;
    for (int t = 0; t < T; t++)
        for (int m = 0; m < H; m++) {
            double acc = L->n_shared ? y_shared[(size_t)t * H + m] : 0.0;
            for (int j = 0; j < k; j++)
                if (topk_idx[(size_t)t * k + j] >= 0)
                    acc += (double)topk_w[(size_t)t * k + j] * y_assign[((size_t)t * k + j) * H + m];
            y[(size_t)t * H + m] = acc;
        }
}

/* Batched driver: group the assignments by expert and apply every unique expert
 * once, to all the tokens routed to it. */
void orc_forward(const orc_layer *L, const uint16_t *x, int T, const float *logits_in,
                 orc_result *R)
{
    int H = L->H, k = L->k, E = L->E;
    double *xd = (double *)malloc(sizeof(double) * (size_t)T * H);
    decode_tokens(x, T, H, xd);
    route_all(L, x, T, logits_in, R);
    orc_group(R->topk_idx, T, k, E, R->counts, R->offsets, R->perm, R->unique, &R->n_unique);
    for (int ui = 0; ui < R->n_unique; ui++) {
        int e = R->unique[ui];
        for (int p = R->offsets[e]; p < R->offsets[e + 1]; p++) {
            int a = R->perm[p], t = a / k;
            orc_routed_expert(L, e, xd + (size_t)t * H,
                              R->h_assign ? R->h_assign + (size_t)a * L->I : NULL,
                              R->y_assign + (size_t)a * H);
        }
    }
    if (L->n_shared)
        for (int t = 0; t < T; t++)
            orc_shared_expert(L, xd + (size_t)t * H,
                              R->h_shared ? R->h_shared + (size_t)t * L->I_sh : NULL,
                              R->y_shared + (size_t)t * H);
    combine(L, T, R->y_assign, R->y_shared, R->topk_idx, R->topk_w, R->y);
    free(xd);
}

/* Per-token driver: every token visits its own k experts in order j = 0..k-1. */
void orc_forward_per_token(const orc_layer *L, const uint16_t *x, int T, const float *logits_in,
                           orc_result *R)
{
    int H = L->H, k = L->k, E = L->E;
    double *xd = (double *)malloc(sizeof(double) * (size_t)T * H);
    decode_tokens(x, T, H, xd);
    route_all(L, x, T, logits_in, R);
    orc_group(R->topk_idx, T, k, E, R->counts, R->offsets, R->perm, R->unique, &R->n_unique);
    for (int t = 0; t < T; t++) {
        for (int j = 0; j < k; j++) {
            int a = t * k + j;
            if (R->topk_idx[a] < 0) continue;   /* dropped by top-p */
            orc_routed_expert(L, R->topk_idx[a], xd + (size_t)t * H,
                              R->h_assign ? R->h_assign + (size_t)a * L->I : NULL,
                              R->y_assign + (size_t)a * H);
        }
        if (L->n_shared)
            orc_shared_expert(L, xd + (size_t)t * H,
                              R->h_shared ? R->h_shared + (size_t)t * L->I_sh : NULL,
                              R->y_shared + (size_t)t * H);
    }
    combine(L, T, R->y_assign, R->y_shared, R->topk_idx, R->topk_w, R->y);
    free(xd);
}

/* One token's output, for sampled checks at full size: routes token t of x
 * (using logits_in row t when given) and evaluates only that token. */
void orc_forward_token(const orc_layer *L, const uint16_t *x_t, const float *logits_t,
                       int32_t *topk_idx, float *topk_w, float *gap, double *y)
{
    int H = L->H, k = L->k, E = L->E;
    float *logits = (float *)malloc(sizeof(float) * (size_t)E);
    if (logits_t) memcpy(logits, logits_t, sizeof(float) * (size_t)E);
    else orc_router_logits(x_t, 1, H, L->Wr, E, logits);
    orc_route_p(logits, L->bias, 1, E, k, L->scaling, L->top_p, topk_idx, topk_w, NULL, gap);
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *ye = (double *)malloc(sizeof(double) * (size_t)H);
    decode_tokens(x_t, 1, H, xd);
    for (int m = 0; m < H; m++) y[m] = 0.0;
    if (L->n_shared) orc_shared_expert(L, xd, NULL, y);
    for (int j = 0; j < k; j++) {
        if (topk_idx[j] < 0) continue;   /* dropped by top-p */
        orc_routed_expert(L, topk_idx[j], xd, NULL, ye);
        for (int m = 0; m < H; m++) y[m] += (double)topk_w[j] * ye[m];
    }
    free(logits);
    free(xd);
    free(ye);
}
