// moe_router.cu -- router GEMV, sigmoid scores, top-k, combine weights and the
// per-expert grouping of assignments.
//
// Router: DeepSeek-V3-style sigmoid router ("Show HN: 低速のコンピュータでGLM 5.2を
// 動かす方法", section 実装済み機能): logits from fp32 router weights and fp16 tokens
// with fp32 accumulation; s = sigmoid(logit) evaluated in fp64 and rounded to fp32;
// selection score s + bias in fp32; the k best (ties -> lower expert index); weights
// scaling * s_j / sum s.  The bias only selects.
// Grouping: the batch MoE union of the same page (each unique expert read once for all
// its tokens), in a fixed, deterministic order ("GLM-5.3-Flash 320B MoEを4枚のCMP
// 170HXで動かすvLLMレシピ", section "Ampere世代のGPU向けに最適化された独自カーネル群").
//
// One launch serves moe_forward: CTAs (expert group, token tile) compute logits; the
// last CTA to finish a token tile runs that tile's top-k; the last tile to finish runs
// the grouping.  Counters are reset by the CTA that consumes them (atomicInc wraps).
#include <cuda_fp16.h>
#include <math.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kRouterThreads = 256;
constexpr int kMaxEpc = 4;

__device__ __forceinline__ float sigmoid_ref(float logit)
{
    return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(logit))));
}

// ---------------------------------------------------------------------------- top-k
// One warp per token: k rounds of a warp-wide argmax over the selection scores.
__device__ void topk_token(const float *logits_row, const float *bias, int E, int k,
                           float scaling, int32_t *idx_out, float *w_out)
{
    const int lane = threadIdx.x & 31;
    constexpr int kPer = kMaxExperts / 32;
    float sel[kPer];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        sel[i] = -INFINITY;
        if (e < E) sel[i] = sigmoid_ref(__ldcg(logits_row + e)) + bias[e];
    }
    int my_idx = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !(taken >> i & 1u) && (be == 0x7fffffff || sel[i] > bv)) {
                bv = sel[i];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            const bool take = (be == 0x7fffffff) ||
                              (oe != 0x7fffffff && (ov > bv || (ov == bv && oe < be)));
            if (take) {
                bv = ov;
                be = oe;
            }
        }
        if (be != 0x7fffffff && (be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) my_idx = be;
    }
    // combine weights from the unbiased scores, summed in order j = 0..k-1
    double s_mine = 0.0;
    if (lane < k) s_mine = static_cast<double>(sigmoid_ref(__ldcg(logits_row + my_idx)));
    double sum = 0.0;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, s_mine, j);
    if (lane < k) {
        idx_out[lane] = my_idx;
        w_out[lane] = static_cast<float>(static_cast<double>(scaling) * (s_mine / sum));
    }
}

// ---------------------------------------------------------------------------- grouping
// Single-warp stable counting sort of the T*k assignment ids by expert.
__device__ void group_warp(const int32_t *topk_idx, int n, int E, int32_t *counts,
                           int32_t *offsets, int32_t *perm, int32_t *unique, int32_t *n_unique,
                           int *sm_run, int *sm_off, int *status)
{
    const int lane = threadIdx.x & 31;
    for (int e = lane; e < E; e += 32) sm_run[e] = 0;
    __syncwarp();
    // pass 1: counts
    for (int base = 0; base < n; base += 32) {
        const int a = base + lane;
        int e = (a < n) ? __ldcg(topk_idx + a) : -1;
        if (a < n && (e < 0 || e >= E)) {
            record_error(status, MOE_ERR_DEVICE_BOUNDS);
            e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) sm_run[e] += __popc(peers);
        __syncwarp();
    }
    // exclusive scan of counts -> offsets
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
        const int e = base + lane;
        const int c = (e < E) ? sm_run[e] : 0;
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (e < E) {
            counts[e] = c;
            offsets[e] = carry + incl - c;
            sm_off[e] = carry + incl - c;
        }
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        offsets[E] = carry;
        sm_off[E] = carry;
    }
    __syncwarp();
    // unique experts, ascending
    int nu = 0;
    for (int base = 0; base < E; base += 32) {
        const int e = base + lane;
        const bool has = e < E && sm_run[e] > 0;
        const unsigned b = __ballot_sync(0xffffffffu, has);
        if (has) unique[nu + __popc(b & ((1u << lane) - 1u))] = e;
        nu += __popc(b);
    }
    if (lane == 0) *n_unique = nu;
    __syncwarp();
    for (int e = lane; e < E; e += 32) sm_run[e] = 0;
    __syncwarp();
    // pass 2: place every assignment, ascending a inside its expert
    for (int base = 0; base < n; base += 32) {
        const int a = base + lane;
        int e = (a < n) ? __ldcg(topk_idx + a) : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) {
            const int rank = __popc(peers & ((1u << lane) - 1u));
            perm[sm_off[e] + sm_run[e] + rank] = a;
        }
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) sm_run[e] += __popc(peers);
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------- kernels
__global__ void __launch_bounds__(kRouterThreads) router_kernel(RouterParams p)
{
    __shared__ float red[kRouterThreads / 32][kMaxEpc * kRouterTokTile];
    __shared__ int s_flag;
    __shared__ int sm_run[kMaxExperts];
    __shared__ int sm_off[kMaxExperts + 1];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tt = blockIdx.y;
    const int t0 = tt * kRouterTokTile;
    const int nt = min(kRouterTokTile, p.T - t0);

    if (p.do_gemv) {
        const int e0 = blockIdx.x * p.experts_per_cta;
        const int ne = min(p.experts_per_cta, p.E - e0);
        float acc[kMaxEpc][kRouterTokTile];
#pragma unroll
        for (int i = 0; i < kMaxEpc; ++i)
#pragma unroll
            for (int t = 0; t < kRouterTokTile; ++t) acc[i][t] = 0.f;
        const int H4 = p.H >> 2;
        for (int h4 = tid; h4 < H4; h4 += kRouterThreads) {
            float4 wv[kMaxEpc];
#pragma unroll
            for (int i = 0; i < kMaxEpc; ++i)
                if (i < ne) wv[i] = __ldg(reinterpret_cast<const float4 *>(p.w + (size_t)(e0 + i) * p.H) + h4);
#pragma unroll
            for (int t = 0; t < kRouterTokTile; ++t) {
                if (t < nt) {
                    const uint2 xr = __ldg(reinterpret_cast<const uint2 *>(p.x + (size_t)(t0 + t) * p.H) + h4);
                    const float2 xa = __half22float2(*reinterpret_cast<const __half2 *>(&xr.x));
                    const float2 xb = __half22float2(*reinterpret_cast<const __half2 *>(&xr.y));
#pragma unroll
                    for (int i = 0; i < kMaxEpc; ++i)
                        if (i < ne) {
                            float a = acc[i][t];
                            a = fmaf(wv[i].x, xa.x, a);
                            a = fmaf(wv[i].y, xa.y, a);
                            a = fmaf(wv[i].z, xb.x, a);
                            a = fmaf(wv[i].w, xb.y, a);
                            acc[i][t] = a;
                        }
                }
            }
        }
        // deterministic block reduction: butterfly inside warps, then warps in order
#pragma unroll
        for (int i = 0; i < kMaxEpc; ++i)
#pragma unroll
            for (int t = 0; t < kRouterTokTile; ++t) {
                float v = acc[i][t];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) red[warp][i * kRouterTokTile + t] = v;
            }
        __syncthreads();
        if (tid < p.experts_per_cta * kRouterTokTile) {
            const int i = tid / kRouterTokTile, t = tid % kRouterTokTile;
            if (i < ne && t < nt) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kRouterThreads / 32; ++w) v += red[w][tid];
                p.logits[(size_t)(t0 + t) * p.E + e0 + i] = v;
            }
        }
        // last CTA of this token tile runs its top-k
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            const unsigned old = atomicInc(p.tile_counters + tt, gridDim.x - 1);
            s_flag = (old == gridDim.x - 1);
        }
        __syncthreads();
        if (!s_flag) return;
        __threadfence();
    }

    const float *logits = p.do_gemv ? p.logits : p.logits_in;
    for (int t = warp; t < nt; t += kRouterThreads / 32)
        topk_token(logits + (size_t)(t0 + t) * p.E, p.bias, p.E, p.k, p.scaling,
                   p.topk_idx + (size_t)(t0 + t) * p.k, p.topk_w + (size_t)(t0 + t) * p.k);
    if (p.logits_in && p.logits && tid < 32) {   // copy given logits when asked to
        for (int i = lane; i < nt * p.E; i += 32)
            p.logits[(size_t)t0 * p.E + i] = p.logits_in[(size_t)t0 * p.E + i];
    }
    if (!p.do_group) return;

    // last token tile runs the grouping
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned old = atomicInc(p.group_counter, gridDim.y - 1);
        s_flag = (old == gridDim.y - 1);
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    if (warp == 0)
        group_warp(p.topk_idx, p.T * p.k, p.E, p.counts, p.offsets, p.perm, p.unique,
                   p.n_unique, sm_run, sm_off, p.status);
}

__global__ void __launch_bounds__(32) group_kernel(GroupParams p)
{
    __shared__ int sm_run[kMaxExperts];
    __shared__ int sm_off[kMaxExperts + 1];
    group_warp(p.topk_idx, p.T * p.k, p.E, p.counts, p.offsets, p.perm, p.unique, p.n_unique,
               sm_run, sm_off, p.status);
}

__global__ void __launch_bounds__(256) combine_kernel(CombineParams p)
{
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)p.T * p.H) return;
    const int t = static_cast<int>(i / p.H), m = static_cast<int>(i % p.H);
    float acc = p.n_shared ? p.y_shared[i] : 0.f;
    for (int j = 0; j < p.k; ++j)
        acc = fmaf(p.topk_w[(size_t)t * p.k + j], p.y_assign[((size_t)t * p.k + j) * p.H + m], acc);
    p.y[i] = __half_as_ushort(__float2half_rn(acc));
}

// ---------------------------------------------------------------------------- launchers
cudaError_t launch_router(const RouterParams &p, int grid_x, int grid_y, cudaStream_t s)
{
    router_kernel<<<dim3(grid_x, grid_y), kRouterThreads, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_group(const GroupParams &p, cudaStream_t s)
{
    group_kernel<<<1, 32, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_combine(const CombineParams &p, cudaStream_t s)
{
    const size_t n = (size_t)p.T * p.H;
    combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
