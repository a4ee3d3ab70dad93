// moe_api.cu -- the C ABI declared in include/moe.h: validation, TMA descriptors over
// the caller's weights, workspace layout and the launch sequence of each entry point.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>

#include "moe_internal.h"

namespace moe {
cudaError_t launch_router(const RouterParams &p, bool pdl, cudaStream_t s);
cudaError_t router_prepare();
cudaError_t launch_group(const GroupParams &p, cudaStream_t s);
cudaError_t static_route_scratch(void **ptr);
cudaError_t launch_combine(const CombineParams &p, bool pdl, cudaStream_t s);
cudaError_t launch_host_x(const void *src, void *dst, size_t bytes, cudaStream_t s);
cudaError_t launch_x_limbs(const uint16_t *x, int T, int H, unsigned char *limbs, float *scale, cudaStream_t s);
cudaError_t launch_ffn(const LayerMaps &maps, const FfnParams &p, bool gate_up, int ks, int grid, bool pdl,
                       cudaStream_t s);
cudaError_t ffn_prepare(int fmt, int E, int occ[2][2][2]);
cudaError_t tc_prepare(int E);
cudaError_t launch_tc(const LayerMaps &maps, const FfnParams &p, bool gate_up, int grid, bool pdl, cudaStream_t s);
int tc_tokens(const FfnParams &p);
cudaError_t launch_wait_timeout(int *status, unsigned long long max_iters, cudaStream_t s);
cudaError_t fused_prepare(int fmt, int *blocks_per_sm);
cudaError_t launch_fused(const LayerMaps &maps, const FusedParams &p, int grid, bool pdl, cudaStream_t s);

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t up256(size_t v) { return (v + 255) & ~size_t(255); }

// ------------------------------------------------------------------ workspace layout
// The counter block sits first and depends only on the handle, so counters keep their
// place (and their zero value) whatever T successive calls use.
struct Ws {
    size_t ctr_tiles, ctr_group, ctr_work, ctr_chunks, h_amax, f_ctl, f_chunk_ctr, f_chunk_flag, f_tile_ctr, zrow,
        ctr_end;
    size_t logits, score, sel, topk_idx, topk_w, counts, offsets, perm, unique, n_unique, slots;
    size_t x_perm, h, h_sh, y_assign, y_shared, x_stage, y_stage;
    size_t x_limbs, x_limb_scale, h_limbs, h_limb_scale, hsh_limbs, hsh_limb_scale, total;
};

// bytes of one row of int8 limbs of a K-long operand (blocks of 256 values, 3 limbs)
size_t limb_row_bytes(int K) { return (size_t)((K + kLimbBlockK - 1) / kLimbBlockK) * kLimbBlockBytes; }

// Batches that average at most kFewTokensPerExpert tokens per routed expert (T k <= 6 E)
// keep the 8-token items of the int8 path: each weight byte is read once per 8 tokens of
// an expert, and its mma.sync work shrinks with the tokens.  The tensor-memory kernel
// issues the same MMAs per weight byte however few tokens an item holds, so it pays only
// with more tokens per expert.  Measured on B200 (H=6144, I=2048, E=256, top-8, int4), layer
// time int8 path vs tensor-memory kernel: T=32 (1 token per expert) 526 vs 926 us, T=128
// 1087 vs 1394, T=192 (6) 1431 vs 1521, T=256 (8) 1768 vs 1641, T=512 3135 vs 2306.
constexpr long kFewTokensPerExpert = 6;

bool few_tokens_per_expert(const moe_layer_desc &d, int T)
{
    return (long)T * d.top_k <= kFewTokensPerExpert * d.n_experts;
}

// Larger int4 batches with more tokens per expert run the tensor-memory kernel (items of
// 128 rows and 32 or 64 tokens), which needs row counts that are multiples of 128.
bool use_tc(const moe_layer_desc &d, int T)
{
    return d.format == MOE_FMT_INT4_ROWSCALE && T > 16 && !few_tokens_per_expert(d, T) && d.hidden % 128 == 0 &&
           d.inter % 128 == 0 && (!d.n_shared || d.inter_shared % 128 == 0);
}

// the int4 expert kernels run on the int8 path (activations as limbs) for decode-sized
// batches and batches of few tokens per expert (8-token items) and on the tensor-memory
// kernel; int8 and int2 weights run the 8-token int8 path at every batch size
bool use_limbs(const moe_layer_desc &d, int T)
{
    if (d.format == MOE_FMT_INT8_ROWSCALE || d.format == MOE_FMT_INT2_ROWSCALE) return true;
    return d.format == MOE_FMT_INT4_ROWSCALE && (T <= 16 || few_tokens_per_expert(d, T) || use_tc(d, T));
}

Ws ws_layout(const moe_layer_desc &d, int T)
{
    Ws w;
    size_t o = 0;
    const int max_tiles = (d.max_tokens + kRouterTokTile - 1) / kRouterTokTile;
    w.ctr_tiles = o; o += (size_t)max_tiles * 4;
    w.ctr_group = o; o += 4;
    w.ctr_work = o; o += 4 * 4;
    w.ctr_chunks = o; o += (size_t)d.max_tokens * (d.top_k + 1) * 4;
    w.h_amax = o; o += (size_t)d.max_tokens * (d.top_k + 1) * 4;
    // the one-launch decode layer: control words, per-chunk counters and flags, per-tile
    // counters, each word in a 128-byte line of its own
    o = up256(o);
    const size_t fchunks = (size_t)std::min(d.max_tokens, kFusedMaxT) * (d.top_k + 1);
    w.f_ctl = o; o += 8 * kSyncLine * 4;
    w.f_chunk_ctr = o; o += fchunks * kSyncLine * 4;
    w.f_chunk_flag = o; o += fchunks * kSyncLine * 4;
    w.f_tile_ctr = o; o += (size_t)((d.hidden + 63) / 64) * kSyncLine * 4;
    o = up256(o);
    // a row of zeros read by padding token columns (never written)
    w.zrow = o; o = up256(o + (size_t)std::max(d.hidden, std::max(d.inter, d.inter_shared)) * 2);
    w.ctr_end = o;
    const size_t Tk = (size_t)T * d.top_k;
    w.logits = o; o = up256(o + (size_t)T * d.n_experts * 4);
    w.score = o; o = up256(o + (size_t)T * d.n_experts * 4);
    w.sel = o; o = up256(o + (size_t)T * d.n_experts * 4);
    w.topk_idx = o; o = up256(o + Tk * 4);
    w.topk_w = o; o = up256(o + Tk * 4);
    w.counts = o; o = up256(o + (size_t)d.n_experts * 4);
    w.offsets = o; o = up256(o + (size_t)(d.n_experts + 1) * 4);
    w.perm = o; o = up256(o + Tk * 4);
    w.unique = o; o = up256(o + (size_t)d.n_experts * 4);
    w.n_unique = o; o = up256(o + 4);
    w.slots = o; o = up256(o + (size_t)d.n_experts * 16);
    w.x_perm = o; o = up256(o + (size_t)T * d.hidden * 2);
    w.h = o; o = up256(o + Tk * d.inter * 2);
    w.h_sh = o; o = up256(o + (size_t)T * d.inter_shared * 2 * (d.n_shared ? 1 : 0));
    w.y_assign = o; o = up256(o + Tk * d.hidden * 4);
    w.y_shared = o; o = up256(o + (size_t)T * d.hidden * 4 * (d.n_shared ? 1 : 0));
    w.x_stage = o; o = up256(o + (size_t)T * d.hidden * 2);
    w.y_stage = o; o = up256(o + (size_t)T * d.hidden * 2);
    // limb buffers for every row-scaled layer: a batch of fewer tokens than T may take the
    // int8 path where T does not, and the size for T must serve every smaller batch
    const bool lb = row_scaled(d.format);
    w.x_limbs = o; o = up256(o + (lb ? (size_t)T * limb_row_bytes(d.hidden) : 0));
    w.x_limb_scale = o; o = up256(o + (lb ? (size_t)T * 4 : 0));
    w.h_limbs = o; o = up256(o + (lb ? Tk * limb_row_bytes(d.inter) : 0));
    w.h_limb_scale = o; o = up256(o + (lb ? Tk * 4 : 0));
    w.hsh_limbs = o; o = up256(o + (lb && d.n_shared ? (size_t)T * limb_row_bytes(d.inter_shared) : 0));
    w.hsh_limb_scale = o; o = up256(o + (lb && d.n_shared ? (size_t)T * 4 : 0));
    w.total = o;
    return w;
}

template <typename P>
P *at(void *ws, size_t off) { return reinterpret_cast<P *>(static_cast<char *>(ws) + off); }

// ------------------------------------------------------------------ TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// bytes [experts][rows][row_bytes], box {box_inner bytes, 16 rows, 1 expert}
bool make_map(CUtensorMap *m, const void *base, int row_bytes, int rows, int experts, int box_inner,
              bool swizzle128, int box_rows = kRowTile)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)experts};
    cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * (cuuint64_t)rows};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int validate_desc(const moe_layer_desc *d)
{
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->format < MOE_FMT_INT4_ROWSCALE || d->format > MOE_FMT_INT2_ROWSCALE) return MOE_ERR_INVALID_ARG;
    const int kmul = d->format == MOE_FMT_NVFP4 ? 256 : 64;
    if (d->hidden <= 0 || d->hidden > 16384 || d->hidden % kmul) return MOE_ERR_INVALID_ARG;
    if (d->inter <= 0 || d->inter > 16384 || d->inter % kmul) return MOE_ERR_INVALID_ARG;
    if (d->n_shared != 0 && d->n_shared != 1) return MOE_ERR_INVALID_ARG;
    if (d->n_shared && (d->inter_shared <= 0 || d->inter_shared > 16384 || d->inter_shared % kmul))
        return MOE_ERR_INVALID_ARG;
    if (d->n_experts < 1 || d->n_experts > kMaxExperts) return MOE_ERR_INVALID_ARG;
    if (d->top_k < 1 || d->top_k > kMaxTopK || d->top_k > d->n_experts) return MOE_ERR_INVALID_ARG;
    if (d->max_tokens < 1 || d->max_tokens > 65536) return MOE_ERR_INVALID_ARG;
    if (!(d->routed_scaling == d->routed_scaling)) return MOE_ERR_INVALID_ARG;   // NaN
    if (!(d->top_p >= 0.f)) return MOE_ERR_INVALID_ARG;                          // negative or NaN
    return MOE_OK;
}

int validate_weights(const moe_layer_desc *d, const moe_weights *w)
{
    if (!w) return MOE_ERR_INVALID_ARG;
    const void *req[32];
    int n = 0;
    req[n++] = w->router_w; req[n++] = w->router_bias;
    req[n++] = w->gate; req[n++] = w->up; req[n++] = w->down;
    if (row_scaled(d->format)) {
        req[n++] = w->gate_scale; req[n++] = w->up_scale; req[n++] = w->down_scale;
    } else {
        req[n++] = w->gate_bscale; req[n++] = w->up_bscale; req[n++] = w->down_bscale;
        req[n++] = w->gate_tscale; req[n++] = w->up_tscale; req[n++] = w->down_tscale;
    }
    if (d->n_shared) {
        req[n++] = w->shared_gate; req[n++] = w->shared_up; req[n++] = w->shared_down;
        if (row_scaled(d->format)) {
            req[n++] = w->shared_gate_scale; req[n++] = w->shared_up_scale; req[n++] = w->shared_down_scale;
        } else {
            req[n++] = w->shared_gate_bscale; req[n++] = w->shared_up_bscale; req[n++] = w->shared_down_bscale;
            req[n++] = w->shared_gate_tscale; req[n++] = w->shared_up_tscale; req[n++] = w->shared_down_tscale;
        }
    }
    for (int i = 0; i < n; ++i)
        if (!req[i] || !aligned16(req[i])) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// tokens per expert work item: 8 for decode-sized batches (every format: the decode
// variants with their B rows in shared memory) and wherever the int8 path runs (a bucket
// of more tokens becomes several items), 32 on the f16 path for larger batches
int tok_chunk(const moe_layer_desc &d, int T)   // (the tensor-memory kernel sets its own)
{
    return (T <= 16 || (use_limbs(d, T) && !use_tc(d, T))) ? 8 : kTokChunk;
}

int check_ws(const moe_layer *L, int T, void *ws, size_t bytes)
{
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
    if (bytes < ws_layout(L->desc, T).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }


LayerWeights layer_weights(const moe_layer *L)
{
    LayerWeights lw;
    const moe_weights &w = L->w;
    lw.router_w = w.router_w;
    lw.router_bias = w.router_bias;
    if (L->desc.format == MOE_FMT_NVFP4) {
        lw.g_scale = w.gate_tscale; lw.u_scale = w.up_tscale; lw.d_scale = w.down_tscale;
        lw.sh_g_scale = w.shared_gate_tscale; lw.sh_u_scale = w.shared_up_tscale;
        lw.sh_d_scale = w.shared_down_tscale;
    } else {
        lw.g_scale = w.gate_scale; lw.u_scale = w.up_scale; lw.d_scale = w.down_scale;
        lw.sh_g_scale = w.shared_gate_scale; lw.sh_u_scale = w.shared_up_scale;
        lw.sh_d_scale = w.shared_down_scale;
    }
    return lw;
}

RouterParams router_params(const moe_layer *L, const uint16_t *x, int T, void *ws)
{
    const Ws W = ws_layout(L->desc, T);
    RouterParams p = {};
    p.x = x;
    p.w = L->w.router_w;
    p.bias = L->w.router_bias;
    p.score = at<float>(ws, W.score);
    p.sel = at<float>(ws, W.sel);
    p.tile_counters = at<unsigned int>(ws, W.ctr_tiles);
    p.group_counter = at<unsigned int>(ws, W.ctr_group);
    p.status = L->d_status;
    p.T = T;
    p.H = L->desc.hidden;
    p.E = L->desc.n_experts;
    p.k = L->desc.top_k;
    p.scaling = L->desc.routed_scaling;
    p.top_p = (L->desc.top_p > 0.f && L->desc.top_p < 1.f) ? L->desc.top_p : 0.f;
    return p;
}

FfnParams ffn_params(const moe_layer *L, const uint16_t *x, int T, void *ws)
{
    const Ws W = ws_layout(L->desc, T);
    FfnParams p = {};
    p.T = T;
    p.H = L->desc.hidden;
    p.I = L->desc.inter;
    p.I_sh = L->desc.inter_shared;
    p.E = L->desc.n_experts;
    p.k = L->desc.top_k;
    p.n_shared = L->desc.n_shared;
    p.fmt = L->desc.format;
    p.dk = {0x000F000Fu, 0x00F000F0u, 0x64086408u, 0x64806480u, 0x64086408u, 0x2C002C00u, 0xD480D480u};
    p.tok_chunk = tok_chunk(L->desc, T);
    p.x = x;
    p.xb = x;
    p.xb_perm = 0;
    p.zrow = at<uint16_t>(ws, W.zrow);
    p.wt = layer_weights(L);
    p.h = at<__half>(ws, W.h);
    p.h_sh = at<__half>(ws, W.h_sh);
    p.status = L->d_status;
    p.work = at<unsigned int>(ws, W.ctr_work);
    if (use_limbs(L->desc, T)) {
        p.limbs = 1;
        p.x_limbs = at<unsigned char>(ws, W.x_limbs);
        p.x_limb_scale = at<float>(ws, W.x_limb_scale);
        p.h_limbs = at<unsigned char>(ws, W.h_limbs);
        p.h_limb_scale = at<float>(ws, W.h_limb_scale);
        p.hsh_limbs = at<unsigned char>(ws, W.hsh_limbs);
        p.hsh_limb_scale = at<float>(ws, W.hsh_limb_scale);
        p.chunk_counters = at<unsigned int>(ws, W.ctr_chunks);
        p.h_amax = at<unsigned int>(ws, W.h_amax);
    }
    return p;
}

// Warp layout of an expert launch: KS = 1 (each warp owns 16 rows over the whole K) when
// its 64-row items fill the persistent grid about as evenly as 16-row items would, else
// KS = 4 (16-row items, K split four ways).  The number of non-empty experts is known
// only on the device, so the bound min(E, T*k) is used.
struct Launch {
    int ks, grid;
};

Launch ffn_launch(const moe_layer *L, int T, bool gu)
{
    const moe_layer_desc &d = L->desc;
    const int tc = tok_chunk(d, T);
    const int wide = tc > 8;
    const long slots = (long)std::min<long>(d.n_experts, (long)T * d.top_k);
    const long chunks_sh = (T + tc - 1) / tc;
    const long rows = gu ? d.inter : d.hidden;
    const long rows_sh = gu ? d.inter_shared : d.hidden;
    auto items = [&](int rw) {
        return slots * (rows / (kRowTile * rw)) + (d.n_shared ? (rows_sh / (kRowTile * rw)) * chunks_sh : 0);
    };
    // balance per SM (the CTAs of one SM share its bandwidth): items per SM vs. average
    auto eff = [&](long n) {
        const long per_sm = (n + L->num_sms - 1) / L->num_sms;
        return (double)n / (double)(per_sm * L->num_sms);
    };
    if (use_tc(d, T)) return {1, L->num_sms};                         // one CTA per SM
    if (use_limbs(d, T)) return {1, L->num_sms * L->occ[0][gu][0]};   // the int8 path has KS = 1 only
    const long i1 = items(4), i4 = items(1);
    if (i1 >= L->num_sms && eff(i1) >= 0.85 * eff(i4)) return {1, L->num_sms * L->occ[wide][gu][0]};
    return {4, L->num_sms * L->occ[wide][gu][1]};
}

// The decode-sized layer in one launch (moe_fused.cu): int4 and NVFP4 weights.
bool use_fused(int T) { return T >= 1 && T <= kFusedMaxT; }
bool fused_format(int fmt) { return fmt == MOE_FMT_INT4_ROWSCALE || fmt == MOE_FMT_NVFP4; }

int run_fused(const moe_layer *L, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s,
              void *const *events)
{
    const moe_layer_desc &d = L->desc;
    const Ws W = ws_layout(d, T);
    FusedParams p = {};
    p.dk = {0x000F000Fu, 0x00F000F0u, 0x64086408u, 0x64806480u, 0x64086408u, 0x2C002C00u, 0xD480D480u};
    p.T = T;
    p.H = d.hidden;
    p.I = d.inter;
    p.I_sh = d.inter_shared;
    p.E = d.n_experts;
    p.k = d.top_k;
    p.n_shared = d.n_shared;
    p.fmt = d.format;
    p.scaling = d.routed_scaling;
    p.top_p = (d.top_p > 0.f && d.top_p < 1.f) ? d.top_p : 0.f;
    p.x = x;
    p.y = y;
    p.wt = layer_weights(L);
    p.logits = at<float>(ws, W.logits);
    p.score = at<float>(ws, W.score);
    p.sel = at<float>(ws, W.sel);
    p.topk_idx = at<int32_t>(ws, W.topk_idx);
    p.topk_w = at<float>(ws, W.topk_w);
    p.counts = at<int32_t>(ws, W.counts);
    p.offsets = at<int32_t>(ws, W.offsets);
    p.perm = at<int32_t>(ws, W.perm);
    p.unique = at<int32_t>(ws, W.unique);
    p.n_unique = at<int32_t>(ws, W.n_unique);
    p.slots = at<int4>(ws, W.slots);
    p.x_limbs = at<unsigned char>(ws, W.x_limbs);
    p.x_limb_scale = at<float>(ws, W.x_limb_scale);
    p.h = at<__half>(ws, W.h);
    p.h_sh = at<__half>(ws, W.h_sh);
    p.h_limbs = at<unsigned char>(ws, W.h_limbs);
    p.h_limb_scale = at<float>(ws, W.h_limb_scale);
    p.hsh_limbs = at<unsigned char>(ws, W.hsh_limbs);
    p.hsh_limb_scale = at<float>(ws, W.hsh_limb_scale);
    p.h_amax = at<unsigned int>(ws, W.h_amax);
    p.y_assign = at<float>(ws, W.y_assign);
    p.y_shared = at<float>(ws, W.y_shared);
    p.zrow = at<uint16_t>(ws, W.zrow);
    p.ctl = at<unsigned int>(ws, W.f_ctl);
    p.chunk_ctr = at<unsigned int>(ws, W.f_chunk_ctr);
    p.chunk_flag = at<unsigned int>(ws, W.f_chunk_flag);
    p.tile_ctr = at<unsigned int>(ws, W.f_tile_ctr);
    p.status = L->d_status;
    const bool pdl = events == nullptr;
    if (events) cudaEventRecordWithFlags(reinterpret_cast<cudaEvent_t>(events[0]), s, cudaEventRecordExternal);
    const cudaError_t e = launch_fused(L->maps, p, L->num_sms * L->occ_fused, pdl, s);
    if (events)
        for (int i = 1; i < 4; ++i)
            cudaEventRecordWithFlags(reinterpret_cast<cudaEvent_t>(events[i]), s, cudaEventRecordExternal);
    return cuda_status(e);
}

int run_forward(const moe_layer *L, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s,
                void *const *events = nullptr)
{
    const bool pdl = events == nullptr;
    auto rec = [&](int i) {
        // external record nodes when captured, so the events also time graph replays
        if (events) cudaEventRecordWithFlags(reinterpret_cast<cudaEvent_t>(events[i]), s, cudaEventRecordExternal);
    };
    rec(0);
    const Ws W = ws_layout(L->desc, T);
    RouterParams rp = router_params(L, x, T, ws);
    rp.logits = at<float>(ws, W.logits);
    rp.topk_idx = at<int32_t>(ws, W.topk_idx);
    rp.topk_w = at<float>(ws, W.topk_w);
    rp.counts = at<int32_t>(ws, W.counts);
    rp.offsets = at<int32_t>(ws, W.offsets);
    rp.perm = at<int32_t>(ws, W.perm);
    rp.unique = at<int32_t>(ws, W.unique);
    rp.n_unique = at<int32_t>(ws, W.n_unique);
    rp.slots = at<int4>(ws, W.slots);
    rp.do_gemv = 1;
    rp.do_group = 1;
    if (use_limbs(L->desc, T)) {
        rp.x_limbs = at<unsigned char>(ws, W.x_limbs);
        rp.x_limb_scale = at<float>(ws, W.x_limb_scale);
    } else if (L->desc.format == MOE_FMT_INT4_ROWSCALE) {
        rp.x_perm = at<uint16_t>(ws, W.x_perm);
    }
    cudaError_t e = launch_router(rp, pdl, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec(1);

    FfnParams fp = ffn_params(L, x, T, ws);
    fp.offsets = rp.offsets;
    fp.perm = rp.perm;
    fp.topk_w = rp.topk_w;
    fp.unique = rp.unique;
    if (rp.x_perm) {
        fp.xb = rp.x_perm;
        fp.xb_perm = 1;
    }
    fp.n_unique = rp.n_unique;
    fp.slots = rp.slots;
    fp.y_assign = at<float>(ws, W.y_assign);
    fp.y_shared = at<float>(ws, W.y_shared);
    fp.y = y;
    const Launch lg = ffn_launch(L, T, true), ld = ffn_launch(L, T, false);
    const bool tc = use_tc(L->desc, T);
    e = tc ? launch_tc(L->maps, fp, true, lg.grid, pdl, s) : launch_ffn(L->maps, fp, true, lg.ks, lg.grid, pdl, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec(2);
    e = tc ? launch_tc(L->maps, fp, false, ld.grid, pdl, s) : launch_ffn(L->maps, fp, false, ld.ks, ld.grid, pdl, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    CombineParams cp = {};
    cp.y_assign = fp.y_assign;
    cp.y_shared = fp.y_shared;
    cp.topk_w = rp.topk_w;
    cp.y = y;
    cp.T = T;
    cp.H = L->desc.hidden;
    cp.k = L->desc.top_k;
    cp.n_shared = L->desc.n_shared;
    e = launch_combine(cp, pdl, s);
    rec(3);
    return cuda_status(e);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int moe_version(void) { return 100; }

const char *moe_status_string(int status)
{
    switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS";
    default: return "MOE_ERR_UNKNOWN";
    }
}

int moe_layer_create(const moe_layer_desc *desc, const moe_weights *weights, moe_layer **out)
{
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = validate_desc(desc);
    if (rc) return rc;
    rc = validate_weights(desc, weights);
    if (rc) return rc;
    moe_layer *L = new (std::nothrow) moe_layer();
    if (!L) return MOE_ERR_CUDA;
    L->desc = *desc;
    L->w = *weights;
    if (cudaGetDevice(&L->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, L->device) != cudaSuccess) {
        delete L;
        return MOE_ERR_CUDA;
    }
    const moe_layer_desc &d = *desc;
    const moe_weights &w = *weights;
    const int H = d.hidden, I = d.inter, Is = d.inter_shared, E = d.n_experts;
    bool ok = true;
    LayerMaps &M = L->maps;
    const int cb = code_bits(d.format);   // code bytes of a K-long row: K * cb / 8
    for (int r4 = 0; r4 < 2 && ok; ++r4) {
        const int br = r4 ? 4 * kRowTile : kRowTile;
        ok = make_map(r4 ? &M.g4 : &M.g, w.gate, H * cb / 8, I, E, 128, true, br) &&
             make_map(r4 ? &M.u4 : &M.u, w.up, H * cb / 8, I, E, 128, true, br) &&
             make_map(r4 ? &M.d4 : &M.d, w.down, I * cb / 8, H, E, 128, true, br);
        if (ok && d.n_shared)
            ok = make_map(r4 ? &M.sh_g4 : &M.sh_g, w.shared_gate, H * cb / 8, Is, 1, 128, true, br) &&
                 make_map(r4 ? &M.sh_u4 : &M.sh_u, w.shared_up, H * cb / 8, Is, 1, 128, true, br) &&
                 make_map(r4 ? &M.sh_d4 : &M.sh_d, w.shared_down, Is * cb / 8, H, 1, 128, true, br);
        if (ok && d.format == MOE_FMT_NVFP4) {
            ok = make_map(r4 ? &M.gb4 : &M.gb, w.gate_bscale, H / 16, I, E, 16, false, br) &&
                 make_map(r4 ? &M.ub4 : &M.ub, w.up_bscale, H / 16, I, E, 16, false, br) &&
                 make_map(r4 ? &M.db4 : &M.db, w.down_bscale, I / 16, H, E, 16, false, br);
            if (ok && d.n_shared)
                ok = make_map(r4 ? &M.sh_gb4 : &M.sh_gb, w.shared_gate_bscale, H / 16, Is, 1, 16, false, br) &&
                     make_map(r4 ? &M.sh_ub4 : &M.sh_ub, w.shared_up_bscale, H / 16, Is, 1, 16, false, br) &&
                     make_map(r4 ? &M.sh_db4 : &M.sh_db, w.shared_down_bscale, Is / 16, H, 1, 16, false, br);
        }
    }
    if (!ok) {
        delete L;
        return MOE_ERR_CUDA;
    }
    bool occ_ok = router_prepare() == cudaSuccess && ffn_prepare(d.format, d.n_experts, L->occ) == cudaSuccess &&
                  (d.format != MOE_FMT_INT4_ROWSCALE || tc_prepare(d.n_experts) == cudaSuccess) &&
                  (!fused_format(d.format) ||
                   (fused_prepare(d.format, &L->occ_fused) == cudaSuccess && L->occ_fused >= 1));
    for (int a = 0; a < 2; ++a)
        for (int b = 0; b < 2; ++b)
            for (int c = 0; c < 2; ++c) occ_ok = occ_ok && L->occ[a][b][c] >= 1;
    if (!occ_ok) {
        delete L;
        return MOE_ERR_CUDA;
    }
    if (cudaMalloc(&L->d_status, 256) != cudaSuccess) {
        delete L;
        return MOE_ERR_CUDA;
    }
    if (cudaMemset(L->d_status, 0, 256) != cudaSuccess) {
        cudaFree(L->d_status);
        delete L;
        return MOE_ERR_CUDA;
    }
    *out = L;
    return MOE_OK;
}

int moe_layer_destroy(moe_layer *L)
{
    if (!L) return MOE_OK;
    cudaFree(L->d_status);
    delete L;
    return MOE_OK;
}

size_t moe_workspace_size(const moe_layer *L, int T)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return 0;
    return ws_layout(L->desc, T).total;
}

int moe_route(const moe_layer *L, const uint16_t *x, int T, const float *logits_in, float *logits_out,
              int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if ((!x && !logits_in) || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (x && !aligned16(x)) return MOE_ERR_INVALID_ARG;
    int rc = check_ws(L, T, ws, ws_bytes);
    if (rc) return rc;
    const Ws W = ws_layout(L->desc, T);
    RouterParams p = router_params(L, x, T, ws);
    p.logits_in = logits_in;
    p.logits = logits_in ? logits_out : (logits_out ? logits_out : at<float>(ws, W.logits));
    p.topk_idx = topk_idx;
    p.topk_w = topk_w;
    p.do_gemv = logits_in ? 0 : 1;
    p.do_group = 0;
    return cuda_status(launch_router(p, false, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_route_static(const moe_layer *L, const uint16_t *x, int T, const float *logits_in, float *logits_out,
                     int32_t *topk_idx, float *topk_w, moe_stream_t stream)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if ((!x && !logits_in) || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (x && !aligned16(x)) return MOE_ERR_INVALID_ARG;
    const int E = L->desc.n_experts;
    if ((T + kRouterTokTile - 1) / kRouterTokTile > kStaticRouteTiles || (size_t)T * E > (size_t)kStaticRouteElems)
        return MOE_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (static_route_scratch(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    RouterParams p = {};
    p.x = x;
    p.w = L->w.router_w;
    p.bias = L->w.router_bias;
    p.tile_counters = at<unsigned int>(scratch, 0);
    p.score = at<float>(scratch, kStaticRouteScore);
    p.sel = at<float>(scratch, kStaticRouteSel);
    p.logits_in = logits_in;
    p.logits = logits_in ? logits_out : (logits_out ? logits_out : at<float>(scratch, kStaticRouteLogits));
    p.topk_idx = topk_idx;
    p.topk_w = topk_w;
    p.status = L->d_status;
    p.T = T;
    p.H = L->desc.hidden;
    p.E = E;
    p.k = L->desc.top_k;
    p.scaling = L->desc.routed_scaling;
    p.top_p = (L->desc.top_p > 0.f && L->desc.top_p < 1.f) ? L->desc.top_p : 0.f;
    p.do_gemv = logits_in ? 0 : 1;
    p.do_group = 0;
    return cuda_status(launch_router(p, false, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_group(const moe_layer *L, const int32_t *topk_idx, int T, int32_t *counts, int32_t *offsets,
              int32_t *perm, int32_t *unique, int32_t *n_unique, void *ws, size_t ws_bytes,
              moe_stream_t stream)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || !unique || !n_unique || (T > 0 && (!topk_idx || !perm)))
        return MOE_ERR_INVALID_ARG;
    int rc = check_ws(L, T, ws, ws_bytes);
    if (rc) return rc;
    GroupParams p = {};
    p.topk_idx = topk_idx;
    p.counts = counts;
    p.offsets = offsets;
    p.perm = perm;
    p.unique = unique;
    p.n_unique = n_unique;
    p.status = L->d_status;
    p.T = T;
    p.k = L->desc.top_k;
    p.E = L->desc.n_experts;
    return cuda_status(launch_group(p, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_expert_ffn(const moe_layer *L, const uint16_t *x, int T, const int32_t *offsets, const int32_t *perm,
                   float *y_assign, float *y_shared, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !aligned16(x) || !offsets || !perm || !y_assign) return MOE_ERR_INVALID_ARG;
    if (L->desc.n_shared && !y_shared) return MOE_ERR_INVALID_ARG;
    int rc = check_ws(L, T, ws, ws_bytes);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    FfnParams fp = ffn_params(L, x, T, ws);
    fp.offsets = offsets;
    fp.perm = perm;
    fp.y_assign = y_assign;
    fp.y_shared = y_shared;
    const Launch lg = ffn_launch(L, T, true), ld = ffn_launch(L, T, false);
    if (fp.limbs && launch_x_limbs(x, T, L->desc.hidden, const_cast<unsigned char *>(fp.x_limbs),
                                   const_cast<float *>(fp.x_limb_scale), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    const bool tc = use_tc(L->desc, T);
    cudaError_t e = tc ? launch_tc(L->maps, fp, true, lg.grid, false, s) : launch_ffn(L->maps, fp, true, lg.ks, lg.grid, false, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(tc ? launch_tc(L->maps, fp, false, ld.grid, true, s)
                          : launch_ffn(L->maps, fp, false, ld.ks, ld.grid, true, s));
}

int moe_combine(const moe_layer *L, const float *y_assign, const float *y_shared, const float *topk_w,
                int T, uint16_t *y, moe_stream_t stream)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y_assign || !topk_w || !y || (L->desc.n_shared && !y_shared)) return MOE_ERR_INVALID_ARG;
    CombineParams p = {};
    p.y_assign = y_assign;
    p.y_shared = y_shared;
    p.topk_w = topk_w;
    p.y = y;
    p.T = T;
    p.H = L->desc.hidden;
    p.k = L->desc.top_k;
    p.n_shared = L->desc.n_shared;
    return cuda_status(launch_combine(p, false, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_forward(const moe_layer *L, const uint16_t *x, int T, uint16_t *y, void *ws, size_t ws_bytes,
                moe_stream_t stream)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !y || !aligned16(x)) return MOE_ERR_INVALID_ARG;
    int rc = check_ws(L, T, ws, ws_bytes);
    if (rc) return rc;
    return run_forward(L, x, T, y, ws, reinterpret_cast<cudaStream_t>(stream));
}

int moe_forward_timed(const moe_layer *L, const uint16_t *x, int T, uint16_t *y, void *ws, size_t ws_bytes,
                      moe_stream_t stream, void *const events[4], int info[2])
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (!events || !events[0] || !events[1] || !events[2] || !events[3]) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !y || !aligned16(x)) return MOE_ERR_INVALID_ARG;
    int rc = check_ws(L, T, ws, ws_bytes);
    if (rc) return rc;
    if (info) {
        info[0] = 3;   // router | gate/up | down + combine
        info[1] = 4;
    }
    return run_forward(L, x, T, y, ws, reinterpret_cast<cudaStream_t>(stream), events);
}

int moe_forward_fused(const moe_layer *L, const uint16_t *x, int T, uint16_t *y, void *ws, size_t ws_bytes,
                      moe_stream_t stream)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!use_fused(T) || !fused_format(L->desc.format)) return MOE_ERR_UNSUPPORTED;
    if (!x || !y || !aligned16(x)) return MOE_ERR_INVALID_ARG;
    int rc = check_ws(L, T, ws, ws_bytes);
    if (rc) return rc;
    return run_fused(L, x, T, y, ws, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

int moe_forward_host(const moe_layer *L, const uint16_t *x_host, int T, uint16_t *y_host, void *ws,
                     size_t ws_bytes, moe_stream_t stream)
{
    if (!L || T < 0 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
    int rc = check_ws(L, T, ws, ws_bytes);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Ws W = ws_layout(L->desc, T);
    const size_t bytes = (size_t)T * L->desc.hidden * 2;
    // page-locked host memory mapped into the device's address space: its device address
    // (else NULL: a staged copy)
    auto mapped = [](const void *h) -> const void * {
        cudaPointerAttributes pa;
        if (cudaPointerGetAttributes(&pa, h) != cudaSuccess) {
            cudaGetLastError();   // (an unknown pointer is not an error here)
            return nullptr;
        }
        return (pa.type == cudaMemoryTypeHost && pa.devicePointer && aligned16(pa.devicePointer)) ? pa.devicePointer
                                                                                                 : nullptr;
    };
    uint16_t *xd = at<uint16_t>(ws, W.x_stage);
    // x: mapped memory is fetched by the first kernel of the launch chain (host_x_kernel:
    // bus reads overlap the previous layer); other memory is copied on the stream
    const void *xm = mapped(x_host);
    const cudaError_t e = xm ? launch_host_x(xm, xd, bytes, s)
                             : cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // y: mapped memory is written by the combine kernel directly; other memory gets a
    // staged device->host copy
    uint16_t *ym = const_cast<uint16_t *>(static_cast<const uint16_t *>(mapped(y_host)));
    if (ym) return run_forward(L, xd, T, ym, ws, s);
    uint16_t *yd = at<uint16_t>(ws, W.y_stage);
    rc = run_forward(L, xd, T, yd, ws, s);
    if (rc) return rc;
    return cuda_status(cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, s));
}

int moe_get_device_status(const moe_layer *L, int *status)
{
    if (!L || !status) return MOE_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, L->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemset(L->d_status, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    *status = v;
    return MOE_OK;
}

int moe_plan(const moe_layer_desc *desc, int T, int plan[3])
{
    if (!plan || validate_desc(desc) != MOE_OK || T < 1 || T > desc->max_tokens) return MOE_ERR_INVALID_ARG;
    const moe_layer_desc &d = *desc;
    if (use_tc(d, T)) {
        FfnParams p = {};
        p.T = T;
        p.k = d.top_k;
        p.E = d.n_experts;
        plan[0] = MOE_PLAN_TENSOR_MEMORY;
        plan[1] = tc_tokens(p);
    } else {
        plan[1] = tok_chunk(d, T);
        plan[0] = plan[1] > 8 ? MOE_PLAN_F16_BATCH : MOE_PLAN_DECODE;
    }
    plan[2] = use_limbs(d, T) ? 1 : 0;
    return MOE_OK;
}

int moe_workspace_routing(const moe_layer *L, int T, moe_ws_routing *out)
{
    if (!L || !out || T < 1 || T > L->desc.max_tokens) return MOE_ERR_INVALID_ARG;
    const Ws W = ws_layout(L->desc, T);
    out->logits = W.logits;
    out->topk_idx = W.topk_idx;
    out->topk_w = W.topk_w;
    out->counts = W.counts;
    out->offsets = W.offsets;
    out->perm = W.perm;
    out->unique = W.unique;
    out->n_unique = W.n_unique;
    return MOE_OK;
}

int moe_debug_wait_timeout(const moe_layer *L, long long max_iters, moe_stream_t stream)
{
    if (!L || max_iters < 1) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_wait_timeout(L->d_status, (unsigned long long)max_iters,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
