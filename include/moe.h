/*
 * moe.h -- C ABI of the W4A16 quantized-expert Mixture-of-Experts decode layer
 *          for NVIDIA B200 (sm_100a).
 *
 * The layer (one call = one MoE layer over T tokens):
 *   1. router:  logit[t,e] = sum_h W_r[e,h] * x[t,h]   (fp32 weights, fp16 activations,
 *               fp32 accumulation)
 *   2. scores:  s = sigmoid(logit); selection score sel = s + bias[e]; the k experts with
 *               the largest sel (descending, equal scores -> lower expert index);
 *               combine weights w_j = routed_scaling * s_j / sum_j' s_j'
 *   3. grouping: the T*k assignments a = t*k + j are grouped by expert so that every
 *               unique expert is read once and applied to all its tokens
 *   4. experts: h = SiLU(x W_g^T) * (x W_u^T) rounded to fp16, y_e = h W_d^T, weights
 *               dequantised inside the matmul, fp32 accumulation
 *   5. combine: y[t] = shared(x_t) + sum_{j=0..k-1} w_tj * y_{e_tj}(x_t), in that order,
 *               stored as fp16.
 *
 * Sources (web pages on W4A16 quantised-expert inference):
 *  - W4A16 = INT4 weights, FP16 activations; custom kernels fusing MoE routing for small
 *    batches; deterministic MoE block order: "GLM-5.3-Flash 320B MoEを4枚のCMP 170HXで
 *    動かすvLLMレシピ" (648news), sections "OpenAI互換APIで動く320BパラメータのMoE構成" and
 *    "Ampere世代のGPU向けに最適化された独自カーネル群".
 *  - DeepSeek-V3-style sigmoid router, shared expert, int4 with per-row scales, batch MoE
 *    union: "Show HN: 低速のコンピュータでGLM 5.2を動かす方法" (hakusoku), section
 *    "実装済み機能".
 *  - NVFP4 weights decoded in registers inside the matmul: "GTX 1070向け35Bパラメータ
 *    MoEモデル推論エンジン公開" (648news), section "VRAMとシステムメモリで重みを分割する
 *    設計" and "用語の注釈" (NVFP4).
 *  - 256 experts of about 19 MB per layer: hakusoku page, section "Colibrì: 消費者PCで
 *    744BパラメータGLM-5.2を動かす革新的エンジン".
 *
 * Conventions for every call below:
 *  - All tensor pointers are DEVICE pointers unless the name ends in _host.  They are
 *    borrowed: the library never frees them.  Weight pointers given to moe_layer_create
 *    must stay valid and unchanged for the life of the handle.
 *  - Activations are fp16 given as their uint16_t bit patterns, row-major [T][H].
 *  - Quantised matrices are row-major with K (the input dimension) contiguous.  4-bit
 *    formats hold two codes per byte, element 2b in the LOW nibble of byte b.  int4 codes
 *    are two's complement in [-8, 7] with one fp32 scale per output row.  int8 codes are
 *    one two's-complement byte per weight, int2 codes four per byte (element 4b + i in
 *    bits 2i..2i+1 of byte b, two's complement in [-2, 1]), each with one fp32 scale per
 *    output row.  NVFP4 codes are E2M1 with one E4M3 (OCP "FN") scale byte per 16
 *    consecutive K elements of a row and one fp32 scale per (expert, matrix).
 *  - Every call except create/destroy/get_device_status is asynchronous on the caller's
 *    stream, allocates nothing and never synchronises the host, so it may be captured in
 *    a CUDA graph.  A non-zero return means nothing was enqueued.
 *  - Errors found on the device (a bounded wait that gave up, an index out of range)
 *    never trap: kernels record a MOE_ERR_* code in the handle's status word and return.
 *    Read it with moe_get_device_status.
 *  - Results are deterministic: the same inputs give bit-identical outputs (no float
 *    atomics, fixed reduction orders).
 */
#ifndef MOE_W4A16_H
#define MOE_W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Compatible with cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st *moe_stream_t;

/* ---------------------------------------------------------------- status codes */
enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,     /* a pointer, size or shape is invalid (host check) */
    MOE_ERR_UNSUPPORTED = 2,     /* valid request this build does not implement */
    MOE_ERR_WORKSPACE = 3,       /* workspace missing, misaligned or too small */
    MOE_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed */
    MOE_ERR_DEVICE_TIMEOUT = 5,  /* a device-side wait exceeded its iteration limit */
    MOE_ERR_DEVICE_BOUNDS = 6    /* a device-side index check failed; access skipped */
};

/* weight formats */
enum {
    MOE_FMT_INT4_ROWSCALE = 0,   /* int4 codes + fp32 scale per output row */
    MOE_FMT_NVFP4 = 1,           /* E2M1 codes + E4M3 per 16 K-elements + fp32 per matrix */
    MOE_FMT_INT8_ROWSCALE = 2,   /* int8 codes + fp32 scale per output row */
    MOE_FMT_INT2_ROWSCALE = 3    /* int2 codes + fp32 scale per output row */
};

/* Shape and hyper-parameters of one layer. */
typedef struct moe_layer_desc {
    int hidden;            /* H: model width, fan-in of gate/up, fan-out of down */
    int inter;             /* I: intermediate width of a routed expert */
    int inter_shared;      /* I_sh: intermediate width of the shared expert */
    int n_experts;         /* E: routed experts, 1..1024 */
    int top_k;             /* k: experts per token, 1..min(E, 32) */
    int n_shared;          /* shared experts: 0 or 1 */
    float routed_scaling;  /* multiplies the normalised combine weights (e.g. 2.5) */
    int format;            /* MOE_FMT_* */
    int max_tokens;        /* largest T any call on this handle will pass, >= 1 */
    float top_p;           /* adaptive expert top-p: in (0, 1), of each token's k chosen experts
                              only the fewest with the highest scores s whose summed s reaches
                              top_p of the k's sum are kept (at least one), listed first in
                              top-k order with weights renormalised to routed_scaling; the
                              other entries are index -1, weight 0 and reach no expert.
                              0 or >= 1: plain top-k.  (The pages name the option, the
                              "--topp" flag of the hakusoku page's section
                              "実行・チューニングパラメータ", not its rule; this is the reading.)
                              Negative or NaN: MOE_ERR_INVALID_ARG. */
} moe_layer_desc;

/* Device pointers to one layer's parameters (borrowed; see conventions).
 * Routed tensors have a leading expert dimension E; shared ones do not.
 *   router_w     fp32 [E][H]              router_bias fp32 [E]
 *   gate, up     u8   [E][I][H*b/8]       down        u8   [E][H][I*b/8]
 *          (b = bits per code: 4 for int4 and NVFP4, 8 for int8, 2 for int2)
 *   int4, int8, int2: gate_scale, up_scale fp32 [E][I];  down_scale fp32 [E][H]
 *   NVFP4: gate_bscale, up_bscale u8 [E][I][H/16]; down_bscale u8 [E][H][I/16];
 *          gate_tscale, up_tscale, down_tscale fp32 [E]
 *   shared_*: the same without E, with I_sh rows (gate/up) or I_sh*b/8 bytes (down);
 *          shared NVFP4 tensor scales are fp32 [1].
 * Pointers that the chosen format or n_shared does not use may be NULL.  Every pointer
 * must be 16-byte aligned. */
typedef struct moe_weights {
    const float *router_w;
    const float *router_bias;
    const uint8_t *gate, *up, *down;
    const float *gate_scale, *up_scale, *down_scale;
    const uint8_t *gate_bscale, *up_bscale, *down_bscale;
    const float *gate_tscale, *up_tscale, *down_tscale;
    const uint8_t *shared_gate, *shared_up, *shared_down;
    const float *shared_gate_scale, *shared_up_scale, *shared_down_scale;
    const uint8_t *shared_gate_bscale, *shared_up_bscale, *shared_down_bscale;
    const float *shared_gate_tscale, *shared_up_tscale, *shared_down_tscale;
} moe_weights;

typedef struct moe_layer moe_layer;   /* opaque handle */

/* ---------------------------------------------------------------- lifetime */

/* Source: the layer's shape and weight formats -- int8, int4 and int2 with per-row scales
 * (hakusoku page "Show HN: 低速のコンピュータでGLM 5.2を動かす方法", section "実装済み機能"), NVFP4
 * (648news page "GTX 1070向け35BパラメータMoEモデル推論エンジン公開", section "用語の注釈"),
 * 256 experts of about 19 MB (hakusoku page, section "Colibrì: ...").
 * Validates desc and weights and builds the handle: TMA descriptors over the caller's
 * weights and a device status word (the only allocation the library makes).
 * Requirements: H and I (and I_sh) multiples of 64 (int4, int8, int2) or 256 (NVFP4) -- the NVFP4
 * block-scale rows must be 16-byte multiples -- H <= 16384, I, I_sh <= 16384,
 * 1 <= E <= 1024, 1 <= k <= min(E, 32), n_shared in {0, 1}, 1 <= max_tokens <= 65536,
 * all pointers 16-byte aligned.  Uses the current CUDA device.
 * Returns MOE_OK and *out, or an error code and *out = NULL. */
int moe_layer_create(const moe_layer_desc *desc, const moe_weights *weights, moe_layer **out);

/* Source: none of the pages has a handle; this ends the lifetime moe_layer_create began.
 * Frees the handle (and its status word).  The caller must ensure no call on it is
 * still running on the GPU.  NULL is accepted. */
int moe_layer_destroy(moe_layer *layer);

/* Source: none of the pages sizes buffers; the workspace holds the intermediate results of
 * the steps the pages name (logits, top-k, grouping, h, per-expert outputs).
 * Bytes of device workspace any call with T tokens needs (0 if T is out of range).
 * One workspace serves every entry point; it must be 256-byte aligned, and must not be
 * used by two calls that may run concurrently.  It holds a few completion counters that
 * must be ZERO before the workspace's first use (one cudaMemset of the whole buffer);
 * every call leaves them at zero again.  After a device-side error
 * (moe_get_device_status != MOE_OK) zero it again before reuse. */
size_t moe_workspace_size(const moe_layer *layer, int T);

/* ---------------------------------------------------------------- staged steps */

/* Source: DeepSeek-V3-style sigmoid router with a selection bias (hakusoku page, section
 * "実装済み機能"); routing fused into the small-batch kernels (648news GLM-5.3-Flash vLLM
 * page, section "Ampere世代のGPU向けに最適化された独自カーネル群").
 * Steps 1-2.  x [T][H] fp16.  If logits_in is non-NULL ([T][E] fp32) the router GEMV is
 * skipped and these logits are used (bit-exact selection from given logits).  If
 * logits_out is non-NULL the fp32 logits are written there.  Outputs: topk_idx int32
 * [T][k] (descending selection score), topk_w fp32 [T][k].  With the layer's adaptive
 * top-p active, each token's kept experts come first (in that order) and the remaining
 * entries are index -1 with weight 0.  0 <= T <= max_tokens. */
int moe_route(const moe_layer *layer, const uint16_t *x, int T, const float *logits_in,
              float *logits_out, int32_t *topk_idx, float *topk_w, void *workspace,
              size_t workspace_bytes, moe_stream_t stream);

/* moe_route without a workspace: the same kernel and the same results (bit-exact
 * topk_idx and topk_w), with its scratch in a fixed static device array of the library
 * (256 B of counters + 3 x 16384 floats, 196864 bytes, per device) instead of a caller
 * buffer.  There is no counterpart in the method's sources: it is a convenience of this
 * library for callers that have no workspace to pass and must not allocate, such as an
 * engine that has already handed every free byte of the device to its KV cache, or a
 * latency-critical loop in which the implicit device-wide synchronisation of
 * cudaMalloc/cudaFree would stall the other streams.  This call allocates nothing; it
 * makes no cudaMalloc, cudaFree or allocating library call.
 * Limits: ceil(T / 16) <= 64 and T * n_experts <= 16384 (e.g. T <= 64 with 256
 * experts); larger calls return MOE_ERR_WORKSPACE and launch nothing.  Other arguments
 * and errors as moe_route.
 * The first call in each CUDA context (each device's primary context, or any other
 * context the caller makes current) looks up the array's address there
 * (cudaGetSymbolAddress, which may load the module) and caches it keyed by the context's
 * unique id, so a context created later, e.g. after cudaDeviceReset, gets its own lookup;
 * make that first call before any stream capture begins.
 * The scratch is shared by every handle and stream of the device: calls that may
 * overlap in time (other streams, other threads, other handles) race on it and must be
 * serialised by the caller.  Its 64 tile counters must be zero when a call starts: they
 * are zero at load and every complete call leaves them zero; after a device-side error
 * (moe_get_device_status != MOE_OK) the counters may be left non-zero and this entry
 * point must not be used again in the process. */
int moe_route_static(const moe_layer *layer, const uint16_t *x, int T, const float *logits_in,
                     float *logits_out, int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/* Source: the batch MoE union, each unique expert of a batch read once and applied to all
 * its tokens (hakusoku page, section "実装済み機能"), in a deterministic order (648news
 * GLM-5.3-Flash vLLM page, section "Ampere世代のGPU向けに最適化された独自カーネル群").
 * Step 3.  topk_idx [T][k] with values in [0, E), or -1 for an entry dropped by top-p
 * (other out-of-range values set MOE_ERR_DEVICE_BOUNDS and are dropped too).  Outputs
 * (int32): counts [E], offsets [E+1] (exclusive prefix sum of counts; offsets[E] is the
 * number of grouped assignments), perm [T*k] (the first offsets[E] entries: assignment
 * ids a = t*k + j ordered by expert, ascending a inside an expert), unique [E] (experts
 * with counts > 0, ascending; entries past n_unique are unspecified), n_unique [1]. */
int moe_group(const moe_layer *layer, const int32_t *topk_idx, int T, int32_t *counts,
              int32_t *offsets, int32_t *perm, int32_t *unique, int32_t *n_unique,
              void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* Source: W4A16, int4 weights with fp16 activations (648news GLM-5.3-Flash vLLM page,
 * section "OpenAI互換APIで動く320BパラメータのMoE構成"); weights decoded inside the matmul
 * kernel (648news GTX 1070 page, section "VRAMとシステムメモリで重みを分割する設計"); the
 * always-on shared expert (hakusoku page, section "実装済み機能").
 * Step 4 (and the shared expert).  Uses offsets [E+1] and perm [T*k] as moe_group
 * writes them.  y_assign fp32 [T*k][H]: row a = t*k + j holds expert topk_idx[t][j]
 * applied to x[t] (unscaled).  y_shared fp32 [T][H] receives the shared expert (may be
 * NULL when n_shared = 0). */
int moe_expert_ffn(const moe_layer *layer, const uint16_t *x, int T, const int32_t *offsets,
                   const int32_t *perm, float *y_assign, float *y_shared, void *workspace,
                   size_t workspace_bytes, moe_stream_t stream);

/* Source: the weighted sum of the routed experts plus the shared expert of the
 * DeepSeek-V3-style layer (hakusoku page, section "実装済み機能").
 * Step 5.  y [T][H] fp16 = y_shared[t] + sum_j topk_w[t][j] * y_assign[t*k + j], summed
 * in fp32 in the order shared, j = 0 .. k-1; terms with weight 0 (entries dropped by
 * top-p, whose y_assign rows are never written) are skipped.  y_shared may be NULL when
 * n_shared = 0. */
int moe_combine(const moe_layer *layer, const float *y_assign, const float *y_shared,
                const float *topk_w, int T, uint16_t *y, moe_stream_t stream);

/* ---------------------------------------------------------------- fused layer */

/* Source: the whole MoE layer with routing fused into the small-batch kernels (648news
 * GLM-5.3-Flash vLLM page, section "Ampere世代のGPU向けに最適化された独自カーネル群") and
 * replayed as one unit per decode step (648news GTX 1070 page, section
 * "Pascal世代の制約をCUDAグラフとカーネル最適化で克服").
 * Steps 1-5 in as few launches as the path allows.  x [T][H] fp16 in, y [T][H] fp16
 * out (x and y may not overlap).  Equal within tolerance to the staged path. */
int moe_forward(const moe_layer *layer, const uint16_t *x, int T, uint16_t *y,
                void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* Source: as moe_forward (routing fused into the small-batch kernels, one replayed unit per
 * decode step), taken to one launch.
 * moe_forward for decode-sized batches (1 <= T <= 16) in ONE persistent launch: router
 * GEMV, top-k, grouping, gate/up, down and the combine run as one ordered list of work
 * items, with flags (not grid barriers) between the steps -- the expert weights of the
 * shared expert stream while routing runs, down items of an expert start while other
 * experts' gate/up items still run, and each 64-row output tile is combined by the CTA
 * whose down item completes it.  The routing (logits, top-k, weights, grouping) is the
 * same bits as moe_forward's.  With int4 weights y is moe_forward's y bit for bit (the
 * same exact integer sums, the same epilogue and combine order); with NVFP4 the fp32 sums
 * may run in another order (moe_forward splits K across warps for small layers), within
 * the layer's tolerance.  Returns MOE_ERR_UNSUPPORTED for T > 16 and for int8 or int2
 * weights (and MOE_OK for T = 0).
 * The grid holds two CTAs per SM and its CTAs wait for one another's flags (bounded waits,
 * MOE_ERR_DEVICE_TIMEOUT if one gives up): do not run it beside another kernel that keeps
 * SMs occupied for good. */
int moe_forward_fused(const moe_layer *layer, const uint16_t *x, int T, uint16_t *y,
                      void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* moe_forward with HOST activations: x_host [T][H] in, y_host [T][H] out (fp16 bits);
 * returns once enqueued; synchronise the stream before reading y_host.  Page-locked host
 * memory mapped into the device's address space (any cudaHostAlloc / cudaMallocHost
 * allocation on a system with unified addressing) is read and written by the kernels
 * themselves: the first kernel of the launch chain fetches x over the bus while the
 * previous work on the stream finishes and stores it in the workspace once that work is
 * complete, and the combine kernel writes y_host directly, so the layer keeps its launch
 * chain.  Other host memory is staged with copies on the stream (synchronous for pageable
 * memory).  The workspace's staging buffer is reused by every call: calls that share a
 * workspace must be ordered (the same stream, or one capture sequence). */
int moe_forward_host(const moe_layer *layer, const uint16_t *x_host, int T, uint16_t *y_host,
                     void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- diagnostics */

/* Human-readable name of a MOE_* status code (static storage). */
const char *moe_status_string(int status);

/* Synchronises the device, returns in *status the first device-side error recorded on
 * this handle since the last call (MOE_OK if none) and clears it.  For tests and
 * debugging, not for the hot path. */
int moe_get_device_status(const moe_layer *layer, int *status);

/* Source: none of the pages chooses kernels; the choice is this implementation's (measured
 * crossovers in its design notes).  Which expert kernels (steps 4-6) moe_forward,
 * moe_forward_host and moe_expert_ffn run for a batch of T tokens of a layer with this
 * description:
 *   plan[0]  MOE_PLAN_DECODE (the streaming kernels with 8-token work items: decode-sized
 *            batches, int4 batches of at most 6 tokens per routed expert, int8 and int2 at
 *            every T), MOE_PLAN_F16_BATCH (32-token items on the f16 path: NVFP4 above 16
 *            tokens, int4 shapes the tensor-memory kernel does not take) or
 *            MOE_PLAN_TENSOR_MEMORY (the tcgen05 kernel: int4 above 16 tokens and more than
 *            6 tokens per routed expert, H, I, I_sh multiples of 128);
 *   plan[1]  tokens per work item (8, 32, or 32 / 64 on the tensor-memory kernel);
 *   plan[2]  1 if activations are carried as exact int8 limbs, 0 for f16.
 * A pure host function: no handle, no GPU.  Returns MOE_ERR_INVALID_ARG for an invalid
 * description, a NULL plan or T outside [1, max_tokens]. */
#define MOE_PLAN_DECODE 0
#define MOE_PLAN_F16_BATCH 1
#define MOE_PLAN_TENSOR_MEMORY 2
int moe_plan(const moe_layer_desc *desc, int T, int plan[3]);

/* Where moe_forward (and moe_forward_host) leave the routing and grouping results of a
 * call with T tokens inside its workspace: byte offsets from the workspace's start of
 *   logits fp32 [T][E], topk_idx int32 [T][k], topk_w fp32 [T][k]   (as moe_route
 *                                                 writes them)
 *   counts int32 [E], offsets int32 [E+1], perm int32 [T*k], unique int32 [E],
 *   n_unique int32 [1]                           (as moe_group writes them).
 * The values stay there until the workspace is used by another call.  For tests and
 * debugging (a check that the grouping the fused path runs is the method's grouping),
 * not for the hot path.  Returns MOE_ERR_INVALID_ARG for a NULL argument or T out of
 * [1, max_tokens]. */
typedef struct moe_ws_routing {
    size_t logits, topk_idx, topk_w, counts, offsets, perm, unique, n_unique;
} moe_ws_routing;
int moe_workspace_routing(const moe_layer *layer, int T, moe_ws_routing *out);

/* Test hook for the bounded waits: launches one block whose consumer waits on an
 * mbarrier that nothing completes, with an iteration limit of max_iters.  The kernel
 * gives up, records MOE_ERR_DEVICE_TIMEOUT in the status word and returns. */
int moe_debug_wait_timeout(const moe_layer *layer, long long max_iters, moe_stream_t stream);

/* moe_forward for per-kernel timing: the same kernels on the same work, launched without
 * programmatic dependent launch, with events[0..3] (cudaEvent_t handles, recorded on the
 * stream) between them.  info (may be NULL) receives info[0] = the number of timed parts
 * and info[1] = the number of kernels the call launches.  Three parts: [0, 1] the router,
 * [1, 2] the gate/up kernel, [2, 3] the down kernel and the combine kernel.  One part:
 * [0, 1] the single kernel that runs the whole layer; events[2] and events[3] are
 * recorded right after events[1].  For benchmarks and profiling, not for the hot path. */
int moe_forward_timed(const moe_layer *layer, const uint16_t *x, int T, uint16_t *y,
                      void *workspace, size_t workspace_bytes, moe_stream_t stream,
                      void *const events[4], int info[2]);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_W4A16_H */
