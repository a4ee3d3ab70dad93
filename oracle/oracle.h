/*
 * oracle.h -- plain FP64 CPU reference of the W4A16 quantized-expert MoE layer.
 * TEST INFRASTRUCTURE: used only by the tests, the smoke check and the benchmark's
 * CPU-baseline leg.  Independent of the CUDA path (no shared code or headers).
 *
 * Layouts (all row-major, K contiguous inside a row, two 4-bit codes per byte with
 * element 2b in the low nibble of byte b):
 *   x        uint16 fp16 bit patterns [T][H]
 *   Wr       fp32 [E][H]; bias fp32 [E]
 *   g, u     codes [E][I][H/2];  d codes [E][H][I/2]
 *   int4:    sg, su fp32 [E][I]; sd fp32 [E][H]           (one scale per output row)
 *   NVFP4:   bg, bu E4M3 bytes [E][I][H/16]; bd [E][H][I/16]; tg, tu, td fp32 [E]
 *   shared:  the same without the E dimension and with I_sh rows.
 */
#ifndef ORACLE_H
#define ORACLE_H
#include <stdint.h>

#define ORC_INT4 0
#define ORC_NVFP4 1
#define ORC_INT8 2   /* one two's-complement byte per weight, one fp32 scale per row */
#define ORC_INT2 3   /* four 2-bit two's-complement codes per byte (element 4b+i in bits 2i..2i+1) */

typedef struct {
    int format;                 /* ORC_INT4, ORC_NVFP4, ORC_INT8 or ORC_INT2 */
    int N, K;                   /* output rows, inputs per row */
    const uint8_t *codes;       /* [N][K/2] (int4, NVFP4), [N][K] (int8), [N][K/4] (int2) */
    const float *row_scale;     /* int4, int8, int2: [N] */
    const uint8_t *block_scale; /* NVFP4: [N][K/16] E4M3 */
    float tensor_scale;         /* NVFP4 */
} orc_matrix;

typedef struct {
    int H, I, I_sh, E, k, n_shared, format;
    double scaling;
    const float *Wr, *bias;
    const uint8_t *g, *u, *d;
    const float *sg, *su, *sd;
    const uint8_t *bg, *bu, *bd;
    const float *tg, *tu, *td;
    const uint8_t *sh_g, *sh_u, *sh_d;
    const float *sh_sg, *sh_su, *sh_sd;
    const uint8_t *sh_bg, *sh_bu, *sh_bd;
    float sh_tg, sh_tu, sh_td;
    double top_p;               /* adaptive expert top-p in (0, 1); otherwise off */
} orc_layer;

/* Caller-allocated outputs of a forward pass (h_assign / h_shared may be NULL). */
typedef struct {
    float *logits;      /* [T][E] */
    float *sel;         /* [T][E] selection scores s + b */
    float *gap;         /* [T] k-th minus (k+1)-th selection score */
    int32_t *topk_idx;  /* [T][k] */
    float *topk_w;      /* [T][k] */
    int32_t *counts;    /* [E] */
    int32_t *offsets;   /* [E+1] */
    int32_t *perm;      /* [T*k] */
    int32_t *unique;    /* [E] */
    int32_t n_unique;
    double *h_assign;   /* [T*k][I] or NULL */
    double *h_shared;   /* [T][I_sh] or NULL */
    double *y_assign;   /* [T*k][H] */
    double *y_shared;   /* [T][H] */
    double *y;          /* [T][H] */
} orc_result;

double orc_half_to_double(uint16_t h);
int orc_int4_at(const uint8_t *row, long k);
int orc_int8_at(const uint8_t *row, long k);
int orc_int2_at(const uint8_t *row, long k);
/* Per-row symmetric quantisation of fp32 rows [N][K] to bits = 8, 4 or 2 two's-complement
 * codes, packed as the decoders read them, with one fp32 scale per row (see oracle.c). */
void orc_quantize_rows(const float *w, int N, int K, int bits, uint8_t *codes, float *scale);
double orc_e2m1_to_double(unsigned code);
double orc_e4m3_to_double(uint8_t b);
float orc_sigmoid_f32(float logit);
void orc_dequant_matrix(const orc_matrix *M, double *out);

void orc_router_logits(const uint16_t *x, int T, int H, const float *Wr, int E, float *logits);
void orc_route(const float *logits, const float *bias, int T, int E, int k, double scaling,
               int32_t *topk_idx, float *topk_w, float *sel_out, float *gap_out);
/* The same with adaptive expert top-p: of the k chosen experts only the fewest with the
 * largest scores whose score mass reaches top_p of the k's mass are kept (at least one),
 * listed first in their top-k order and renormalised to the scaling factor; the other
 * entries are index -1, weight 0.  top_p outside (0, 1) is plain top-k. */
void orc_route_p(const float *logits, const float *bias, int T, int E, int k, double scaling,
                 double top_p, int32_t *topk_idx, float *topk_w, float *sel_out, float *gap_out);
void orc_group(const int32_t *topk_idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
               int32_t *perm, int32_t *unique, int32_t *n_unique);
void orc_expert_ffn(const orc_matrix *Wg, const orc_matrix *Wu, const orc_matrix *Wd,
                    const double *x, double *h_out, double *y);
void orc_routed_expert(const orc_layer *L, int e, const double *x, double *h_out, double *y);
void orc_shared_expert(const orc_layer *L, const double *x, double *h_out, double *y);
void orc_forward(const orc_layer *L, const uint16_t *x, int T, const float *logits_in,
                 orc_result *R);
void orc_forward_per_token(const orc_layer *L, const uint16_t *x, int T, const float *logits_in,
                           orc_result *R);
void orc_forward_token(const orc_layer *L, const uint16_t *x_t, const float *logits_t,
                       int32_t *topk_idx, float *topk_w, float *gap, double *y);

#endif
