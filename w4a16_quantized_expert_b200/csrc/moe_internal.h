// moe_internal.h -- parameter blocks shared by the host dispatch and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"
#include "moe_device.cuh"

namespace moe {

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kRouterTokTile = 16;     // tokens per router CTA
constexpr int kFusedMaxT = 16;         // largest batch the one-launch decode layer takes
constexpr int kSyncLine = 32;          // words between two synchronisation words (one 128-byte line each)
constexpr int kRouterMaxDynSmem = 160 * 1024;   // router x staging limit
// scratch of the allocation-free routing entry point: 64 token-tile counters (256 B),
// then score, selection score and logits for up to kStaticRouteElems (token, expert) pairs
constexpr int kStaticRouteTiles = 64;
constexpr int kStaticRouteElems = 16384;
constexpr size_t kStaticRouteScore = 256;
constexpr size_t kStaticRouteSel = kStaticRouteScore + (size_t)kStaticRouteElems * 4;
constexpr size_t kStaticRouteLogits = kStaticRouteSel + (size_t)kStaticRouteElems * 4;
constexpr size_t kStaticRouteBytes = kStaticRouteLogits + (size_t)kStaticRouteElems * 4;
constexpr int kStaticRouteContexts = 64;   // CUDA contexts whose scratch address is cached
constexpr int kRowTile = 16;           // output rows per expert work item (mma M)
constexpr int kTokChunk = 32;          // tokens per expert work item (4 mma N-tiles)

// bits per weight code of a format
__host__ __device__ constexpr int code_bits(int fmt)
{
    return fmt == MOE_FMT_INT8_ROWSCALE ? 8 : fmt == MOE_FMT_INT2_ROWSCALE ? 2 : 4;
}

// formats with one fp32 scale per output row (int8, int4, int2)
__host__ __device__ constexpr bool row_scaled(int fmt) { return fmt != MOE_FMT_NVFP4; }

// Matrices of one layer in one format.  Routed tensors carry a leading expert index.
struct LayerWeights {
    const float *router_w, *router_bias;
    // row scales (int8, int4, int2) or tensor scales (NVFP4), routed [E][rows] / [E], shared
    const float *g_scale, *u_scale, *d_scale;
    const float *sh_g_scale, *sh_u_scale, *sh_d_scale;
};

// TMA descriptors over the quantised weights (3-D: K bytes, rows, experts), with boxes of
// 16 rows (one warp's rows: the K-split launches) and of 64 rows (the four warps' rows of
// a whole-K launch, one copy per matrix and stage).
struct LayerMaps {
    CUtensorMap g, u, d;           // routed codes
    CUtensorMap sh_g, sh_u, sh_d;  // shared codes (expert extent 1)
    CUtensorMap gb, ub, db;        // NVFP4 routed block scales
    CUtensorMap sh_gb, sh_ub, sh_db;
    CUtensorMap g4, u4, d4, sh_g4, sh_u4, sh_d4;          // the same with 64-row boxes
    CUtensorMap gb4, ub4, db4, sh_gb4, sh_ub4, sh_db4;
};

struct RouterParams {
    const uint16_t *x;       // [T][H]
    uint16_t *x_perm;        // optional [T][H]: x with every 8-group in int4 B-fragment order
    unsigned char *x_limbs;  // optional [T][ceil(H/256)][3][256]: x as int8 limbs (needs do_gemv)
    float *x_limb_scale;     // [T] 2^-sh of each row of x_limbs
    const float *w;          // [E][H]
    const float *bias;       // [E]
    const float *logits_in;  // optional [T][E]
    float *logits;           // [T][E] (workspace or caller; may be NULL with logits_in)
    float *score;            // [T][E] sigmoid scores (workspace)
    float *sel;              // [T][E] selection scores s + bias (workspace)
    int32_t *topk_idx;       // [T][k]
    float *topk_w;           // [T][k]
    // grouping outputs (only when do_group)
    int32_t *counts, *offsets, *perm, *unique, *n_unique;
    int4 *slots;             // optional [E]: (expert, count, offset, 0) of the non-empty experts
    unsigned int *tile_counters;  // [ceil(T/16)] expert CTAs done per token tile
    unsigned int *group_counter;  // token tiles whose top-k is done
    int *status;
    int T, H, E, k;
    float scaling;
    float top_p;             // adaptive expert top-p in (0, 1), 0 = off
    int do_gemv, do_group;
    int x_rows, x_bufs;      // GEMV: token rows per shared-memory x buffer, buffers (1 or 2)
};

struct GroupParams {
    const int32_t *topk_idx;
    int32_t *counts, *offsets, *perm, *unique, *n_unique;
    int *status;
    int T, k, E;
};

struct FfnParams {
    DequantK dk;               // int4 dequantisation constants (run-time values on purpose)
    // problem
    int T, H, I, I_sh, E, k, n_shared, fmt;
    const uint16_t *x;         // [T][H]
    const uint16_t *xb;        // x in the B-fragment order of the int4 gate/up kernel, or x
    const uint16_t *zrow;      // max(H, I, I_sh) zero halves (padding token columns)
    int xb_perm;               // xb holds the permuted copy (else int4 gate/up permutes x)
    int tok_chunk;             // tokens per work item: 8 (decode variant) or 32
    int stages, b_stage;       // ring stages and B-row bytes per stage of this launch (set by the launcher)
    unsigned int *work;        // work-item claim counter and finished-CTA counter of this launch
                               // (the caller passes 4: gate/up uses [0..1], down [2..3])
    const int32_t *offsets;    // [E+1]
    const int32_t *perm;       // [T*k]
    const float *topk_w;       // [T][k] (fused combine only)
    const int32_t *unique;     // optional compact list of non-empty experts (router output)
    const int32_t *n_unique;
    const int4 *slots;         // optional: (expert, count, offset) per entry of that list
    LayerWeights wt;
    // intermediate / outputs
    __half *h;                 // [T*k][I], rows in perm order, columns in mma order
    __half *h_sh;              // [T][I_sh]
    float *y_assign;           // [T*k][H]
    float *y_shared;           // [T][H]
    uint16_t *y;               // [T][H] fp16 (fused combine)
    // int8 tensor path (int4 weights, items of <= 8 tokens): activations as int8 limbs
    int limbs;                 // 1: the int4 decode kernels run on the int8 path
    const unsigned char *x_limbs;   // [T][nblk(H)][3][256]
    const float *x_limb_scale;      // [T]
    unsigned char *h_limbs;         // [T*k][nblk(I)][3][256], rows in perm order
    float *h_limb_scale;            // [T*k]
    unsigned char *hsh_limbs;       // [T][nblk(I_sh)][3][256]
    float *hsh_limb_scale;          // [T]
    unsigned int *chunk_counters;   // [T*k + T] gate/up row tiles finished per token chunk
    unsigned int *h_amax;           // [T*k + T] largest |h| of each h row (float bits; reset after use)
    int *status;
};

// The whole decode-sized layer (T <= kFusedMaxT) in one persistent launch (moe_fused.cu).
// Work items, claimed in this order: router tasks (one expert's logits for all T tokens;
// the last one also runs the top-k and the grouping), shared-expert gate/up, routed
// gate/up, shared-expert down, routed down.  Items of 64 output rows and up to 8 tokens.
struct FusedParams {
    DequantK dk;
    int T, H, I, I_sh, E, k, n_shared, fmt;
    float scaling, top_p;
    const uint16_t *x;          // [T][H]
    uint16_t *y;                // [T][H]
    LayerWeights wt;
    float *logits, *score, *sel;                 // [T][E]
    int32_t *topk_idx;                           // [T][k]
    float *topk_w;                               // [T][k]
    int32_t *counts, *offsets, *perm, *unique, *n_unique;
    int4 *slots;                                 // [E]: (expert, count, offset) of the non-empty experts
    unsigned char *x_limbs;                      // int4: [T][nblk(H)][3][256]
    float *x_limb_scale;                         // [T]
    __half *h;                                   // [T*k][I], rows in perm order
    __half *h_sh;                                // [T][I_sh]
    unsigned char *h_limbs, *hsh_limbs;          // int4: limb rows of h and h_sh
    float *h_limb_scale, *hsh_limb_scale;
    unsigned int *h_amax;                        // [T*k + T] largest |h| per row (reset after use)
    float *y_assign;                             // [T*k][H]
    float *y_shared;                             // [T][H]
    const uint16_t *zrow;                        // zero halves (padding rows)
    // Synchronisation words, each alone in its 128-byte line (kSyncLine words apart), so
    // that polling one never queues behind atomics on another.  Control words: [0] epoch of
    // the last complete call, [1] epoch whose routing is published, [2] epoch whose x limbs
    // are complete, [3] router tasks done (wraps), [4] work claims, [5] CTAs done, [6] x-limb
    // tasks done (wraps).
    unsigned int *ctl;
    unsigned int *chunk_ctr;    // [T*k + T] gate/up row tiles done per token chunk (wraps)
    unsigned int *chunk_flag;   // [T*k + T] epoch whose chunk's h (and its limbs) is complete
    unsigned int *tile_ctr;     // [H/64] down items done per output row tile (wraps)
    int *status;
    int stages, stage_bytes, slot_cap;   // ring slots, bytes per slot, slot-table capacity
};

struct CombineParams {
    const float *y_assign, *y_shared, *topk_w;
    uint16_t *y;
    int T, H, k, n_shared;
};

}  // namespace moe

// the opaque handle
struct moe_layer {
    moe_layer_desc desc;
    moe_weights w;
    moe::LayerMaps maps;
    int *d_status;
    int device;
    int num_sms;
    int occ[2][2][2];   // resident CTAs per SM of the expert kernels [tok_chunk 32][gate_up][ks == 4]
    int occ_fused;      // resident CTAs per SM of the one-launch decode-layer kernel
};
