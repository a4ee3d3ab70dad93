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
// One launch serves moe_forward.  CTA (e, tile) computes expert e's logits for a tile of
// up to 16 tokens (every weight load of the row in flight at once), then the sigmoid
// and selection scores.  The last CTA of a tile runs that tile's top-k (a warp per
// token, k rounds of redux.sync max/min on order-preserving keys); the last tile runs
// the grouping.  Counters are reset by the CTA that consumes them (atomicInc wraps).
// The kernel releases its programmatic dependents at once: the expert kernel starts the
// shared expert while routing is still running.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "moe_device.cuh"
#include "moe_internal.h"
#include "moe_route.cuh"

namespace moe {

constexpr int kRouterThreads = 256;
constexpr int kWPerThread = 16;          // float4 of the router row per thread: H <= 16384
constexpr int kRouterXRows = 4;          // token rows per shared-memory x buffer

// ---------------------------------------------------------------------------- grouping
// Single-warp stable counting sort of the T*k assignment ids by expert.
__device__ void group_warp(const int32_t *topk_idx, bool src_smem, int n, int E, int32_t *counts,
                           int32_t *offsets, int32_t *perm, int32_t *unique, int32_t *n_unique,
                           int *sm_run, int *sm_off, int *status, int4 *slots = nullptr)
{
    const int lane = threadIdx.x & 31;
    for (int e = lane; e < E; e += 32) sm_run[e] = 0;
    __syncwarp();
    // pass 1: counts
    for (int base = 0; base < n; base += 32) {
        const int a = base + lane;
        int e = (a < n) ? (src_smem ? topk_idx[a] : __ldcg(topk_idx + a)) : -1;
        if (a < n && (e < -1 || e >= E)) {   // -1: dropped by top-p, no expert
            record_error(status, MOE_ERR_DEVICE_BOUNDS);
            e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) sm_run[e] += __popc(peers);
        __syncwarp();
    }
    // exclusive scan of counts: lane handles experts [lane*P, lane*P + P)
    const int P = (E + 31) >> 5;
    const int e0 = lane * P;
    int local = 0, nz = 0;
    for (int i = 0; i < P; ++i) {
        const int e = e0 + i;
        if (e < E) {
            local += sm_run[e];
            nz += sm_run[e] > 0;
        }
    }
    int incl = local, incl_nz = nz;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        const int u = __shfl_up_sync(0xffffffffu, incl_nz, off);
        if (lane >= off) {
            incl += v;
            incl_nz += u;
        }
    }
    int run = incl - local, ur = incl_nz - nz;
    for (int i = 0; i < P; ++i) {
        const int e = e0 + i;
        if (e < E) {
            const int c = sm_run[e];
            counts[e] = c;
            offsets[e] = run;
            sm_off[e] = run;
            if (c > 0) {
                if (slots) slots[ur] = make_int4(e, c, run, 0);
                unique[ur++] = e;
            }
            run += c;
        }
    }
    if (lane == 31) {
        offsets[E] = incl;
        sm_off[E] = incl;
        *n_unique = incl_nz;
    }
    __syncwarp();
    for (int e = lane; e < E; e += 32) sm_run[e] = 0;
    __syncwarp();
    // pass 2: place every assignment, ascending a inside its expert
    for (int base = 0; base < n; base += 32) {
        const int a = base + lane;
        int e = (a < n) ? (src_smem ? topk_idx[a] : __ldcg(topk_idx + a)) : -1;
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

// ---------------------------------------------------------------------------- one token
// Top-k of a single token by the whole CTA (E <= kRouterThreads, plain top-k): the same
// selection and order as topk_token -- descending selection score, equal scores to the
// lower expert index -- from 64-bit keys (score key, then the complement of the expert
// index), which are all distinct, so every key has one rank.  Each warp first ranks its
// 32 keys among themselves; the k best of every warp are the only candidates, and their
// ranks among the 8k candidates are the final ranks.  Two short passes over shared memory
// replace the k dependent rounds of the one-warp search.  The weights are then formed by
// warp 0 exactly as topk_token forms them.  sK: kRouterThreads 64-bit words; sC: 8k words.
__device__ void topk_one_token_cta(const float *sel_row, const float *score_row, int E, int k, float scaling,
                                   int32_t *idx_out, float *w_out, int *s_topi, float *s_tops,
                                   unsigned long long *sK, unsigned long long *sC, int tid)
{
    const int lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kRouterThreads / 32;
    const bool in = tid < E;
    unsigned long long key = 0ull;
    float sc = 0.f;
    if (in) {
        sc = __ldcg(score_row + tid);
        key = ((unsigned long long)float_key(__ldcg(sel_row + tid)) << 32) | (unsigned)(0xFFFFFFFFu - (unsigned)tid);
    }
    sK[tid] = key;
    for (int j = tid; j < NW * k; j += kRouterThreads) sC[j] = 0ull;
    __syncthreads();
    int r = 0;   // rank inside the warp's 32 keys (absent experts have key 0 and rank last)
#pragma unroll
    for (int j = 0; j < 32; ++j) r += sK[warp * 32 + j] > key;
    const bool cand = in && r < k;
    if (cand) sC[warp * k + r] = key;
    __syncthreads();
    if (cand) {
        int g = 0;
#pragma unroll 16
        for (int j = 0; j < NW * k; ++j) g += sC[j] > key;
        if (g < k) {
            s_topi[g] = tid;
            s_tops[g] = sc;
        }
    }
    __syncthreads();
    if (warp == 0) {
        int my_idx = 0;
        float my_score = 0.f;
        if (lane < k) {
            my_idx = s_topi[lane];
            my_score = s_tops[lane];
        }
        // combine weights from the unbiased scores, summed in order j = 0..k-1
        const double s_mine = lane < k ? static_cast<double>(my_score) : 0.0;
        double sum = 0.0;
#pragma unroll 8
        for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, s_mine, j);
        if (lane < k) {
            idx_out[lane] = my_idx;
            w_out[lane] = static_cast<float>(static_cast<double>(scaling) * (s_mine / sum));
        }
    }
}

// Grouping of a single token's k distinct experts (plain top-k), the results group_block
// gives: the experts in ascending order, one assignment each (perm = their top-k
// positions), counts and offsets of all E experts.  s_topi holds the top-k experts.
__device__ void group_one_token(const int *s_topi, int E, int k, int32_t *counts, int32_t *offsets, int32_t *perm,
                                int32_t *unique, int32_t *n_unique, int4 *slots, int tid)
{
    if (tid < k) {
        const int e = s_topi[tid];
        int r = 0;   // position of e among the k experts in ascending order
#pragma unroll 8
        for (int j = 0; j < k; ++j) r += s_topi[j] < e;
        perm[r] = tid;
        unique[r] = e;
        if (slots) slots[r] = make_int4(e, 1, r, 0);
    }
    if (tid == 0) {
        *n_unique = k;
        offsets[E] = k;
    }
    for (int e = tid; e < E; e += kRouterThreads) {
        int below = 0, has = 0;
#pragma unroll 8
        for (int j = 0; j < k; ++j) {
            const int f = s_topi[j];
            below += f < e;
            has |= f == e;
        }
        counts[e] = has;
        offsets[e] = below;
    }
}

// ---------------------------------------------------------------------------- kernels
__global__ void __launch_bounds__(kRouterThreads) router_kernel(RouterParams p)
{
    extern __shared__ __align__(16) unsigned char r_smem[];   // x rows: [x_bufs][x_rows][H] fp16
    __shared__ float red[kRouterThreads / 32][kRouterTokTile];
    __shared__ float red_max[kRouterThreads / 32][kRouterXRows];
    __shared__ float s_amax[kRouterTokTile];
    __shared__ int s_flag;
    __shared__ __align__(8) int sm_run[kMaxExperts];      // (also the single-token top-k's 64-bit keys)
    __shared__ __align__(8) int sm_off[kMaxExperts + 1];  // (and its candidates)
    __shared__ int s_idx[kRouterTokTile * kMaxTopK];
    __shared__ __align__(8) uint64_t s_bar[2];

    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tt = blockIdx.y;
    const int t0 = tt * kRouterTokTile;
    const int nt = min(kRouterTokTile, p.T - t0);
    if (p.do_gemv) {
        // When launched behind the previous layer (programmatic dependent launch), the
        // router row is pulled into L2 while that work drains (L2 stays coherent, so this
        // is safe whatever the earlier work writes); every load and store of the kernel
        // comes after the wait.
        const char *row = reinterpret_cast<const char *>(p.w + (size_t)blockIdx.x * p.H);
        for (int o = tid * 128; o < p.H * 4; o += kRouterThreads * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(row + o));
    }
    pdl_wait();

    if (p.do_gemv) {
        // ------------------------------------------------ logits of expert e, this tile
        // The expert's fp32 router row is held in registers; the tile's token rows pass
        // through shared memory in groups of x_rows (bulk copies, double-buffered).
        const int e = blockIdx.x;
        const int H4 = p.H >> 2;
        const int R = p.x_rows, NB = p.x_bufs;
        const int ngrp = (nt + R - 1) / R;
        const uint32_t row_bytes = (uint32_t)p.H * 2u;
        const uint16_t *xs = reinterpret_cast<const uint16_t *>(r_smem);
        // CTAs e < ceil(H/256) also write 256-value blocks of x as int8 limbs
        const int nblk = (p.H + kLimbBlockK - 1) / kLimbBlockK;
        const bool conv = p.x_limbs != nullptr && e < nblk;
        if (tid == 0) {
            mbar_init(&s_bar[0], 1);
            mbar_init(&s_bar[1], 1);
            fence_mbar_init();
        }
        __syncthreads();
        auto issue = [&](int g) {   // thread 0: token rows of group g into buffer g % NB
            const int bf = g % NB, r0 = g * R, nr = min(R, nt - r0);
            mbar_arrive_expect_tx(&s_bar[bf], (uint32_t)nr * row_bytes);
            for (int r = 0; r < nr; ++r)
                bulk_copy(r_smem + ((size_t)bf * R + r) * row_bytes, p.x + (size_t)(t0 + r0 + r) * p.H, row_bytes,
                          &s_bar[bf]);
        };
        if (tid == 0)
            for (int g = 0; g < min(NB, ngrp); ++g) issue(g);
        float4 wv[kWPerThread];
#pragma unroll
        for (int j = 0; j < kWPerThread; ++j) {
            const int h4 = j * kRouterThreads + tid;
            wv[j] = (h4 < H4) ? __ldg(reinterpret_cast<const float4 *>(p.w + (size_t)e * p.H) + h4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int g = 0; g < ngrp; ++g) {
            const int bf = g % NB, r0 = g * R, nr = min(R, nt - r0);
            // a wait that gives up records MOE_ERR_DEVICE_TIMEOUT; the CTA still finishes
            mbar_wait(&s_bar[bf], (uint32_t)((g / NB) & 1), p.status);
            float acc[kRouterXRows], amx[kRouterXRows];
#pragma unroll
            for (int r = 0; r < kRouterXRows; ++r) {
                acc[r] = amx[r] = 0.f;
                if (r < nr) {
                    const uint16_t *xrow = xs + ((size_t)bf * R + r) * p.H;
#pragma unroll
                    for (int j = 0; j < kWPerThread; ++j) {
                        const int h4 = j * kRouterThreads + tid;
                        if (h4 < H4) {
                            const uint2 xr = *reinterpret_cast<const uint2 *>(xrow + 4 * h4);
                            const float2 xa = __half22float2(*reinterpret_cast<const __half2 *>(&xr.x));
                            const float2 xb = __half22float2(*reinterpret_cast<const __half2 *>(&xr.y));
                            acc[r] = fmaf(wv[j].x, xa.x, acc[r]);
                            acc[r] = fmaf(wv[j].y, xa.y, acc[r]);
                            acc[r] = fmaf(wv[j].z, xb.x, acc[r]);
                            acc[r] = fmaf(wv[j].w, xb.y, acc[r]);
                            if (conv)
                                amx[r] = fmaxf(amx[r], fmaxf(fmaxf(fabsf(xa.x), fabsf(xa.y)),
                                                             fmaxf(fabsf(xb.x), fabsf(xb.y))));
                        }
                    }
                }
            }
            // deterministic block reduction: butterfly inside warps, then warps in order
#pragma unroll
            for (int r = 0; r < kRouterXRows; ++r) {
                if (r < nr) {
                    float v = acc[r], m = amx[r];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {
                        v += __shfl_xor_sync(0xffffffffu, v, off);
                        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                    }
                    if (lane == 0) {
                        red[warp][r0 + r] = v;
                        red_max[warp][r] = m;
                    }
                }
            }
            __syncthreads();
            if (conv) {
                // the group's rows are in shared memory: their limb blocks b = e (mod gridDim.x)
                if (tid < nr) {
                    float m = 0.f;
#pragma unroll
                    for (int w = 0; w < kRouterThreads / 32; ++w) m = fmaxf(m, red_max[w][tid]);
                    s_amax[r0 + tid] = m;
                }
                __syncthreads();
                const size_t lrow = (size_t)nblk * kLimbBlockBytes;
                for (int b = e; b < nblk; b += gridDim.x)
                    for (int j = tid; j < nr * 32; j += kRouterThreads) {
                        const int r = j >> 5, k8 = (j & 31) * 8, k = b * kLimbBlockK + k8;
                        const uint4 v = k < p.H ? *reinterpret_cast<const uint4 *>(xs + ((size_t)bf * R + r) * p.H + k)
                                                : make_uint4(0u, 0u, 0u, 0u);
                        limb_encode8(v, pow2f(limb_shift(s_amax[r0 + r])),
                                     p.x_limbs + (size_t)(t0 + r0 + r) * lrow + (size_t)b * kLimbBlockBytes, k8);
                    }
                if (e == 0 && tid < nr) p.x_limb_scale[t0 + r0 + tid] = pow2f(-limb_shift(s_amax[r0 + tid]));
                __syncthreads();
            }
            if (p.x_perm && e == 0) {
                // x with every 8-group as (0,4)(1,5)(2,6)(3,7): the B-fragment order of the
                // int4 expert kernels for larger batches, so their inner loop needs no permutes
                const int H8 = p.H >> 3;
                for (int j = tid; j < nr * H8; j += kRouterThreads) {
                    const int r = j / H8, i = j % H8;
                    const uint4 v = *reinterpret_cast<const uint4 *>(xs + ((size_t)bf * R + r) * p.H + 8 * i);
                    reinterpret_cast<uint4 *>(p.x_perm + (size_t)(t0 + r0 + r) * p.H)[i] =
                        make_uint4(pack_lo(v.x, v.z), pack_hi(v.x, v.z), pack_lo(v.y, v.w), pack_hi(v.y, v.w));
                }
                __syncthreads();
            }
            if (tid == 0 && g + NB < ngrp) issue(g + NB);   // the buffer is free again
        }
        if (tid < nt) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kRouterThreads / 32; ++w) v += red[w][tid];
            const size_t o = (size_t)(t0 + tid) * p.E + e;
            const float sc = sigmoid_ref(v);
            p.logits[o] = v;
            p.score[o] = sc;
            p.sel[o] = sc + p.bias[e];
        }
        // the last CTA of this token tile runs its top-k
        __syncthreads();
        if (tid == 0) s_flag = atom_inc_acq_rel(p.tile_counters + tt, gridDim.x - 1) == gridDim.x - 1;
        __syncthreads();
        if (!s_flag) return;
    } else {
        // ------------------------------------------------ scores from given logits
        for (int i = tid; i < nt * p.E; i += kRouterThreads) {
            const size_t o = (size_t)t0 * p.E + i;
            const float l = p.logits_in[o];
            const float sc = sigmoid_ref(l);
            if (p.logits) p.logits[o] = l;
            p.score[o] = sc;
            p.sel[o] = sc + p.bias[i % p.E];
        }
        __syncthreads();
    }

    if (p.T == 1 && p.top_p == 0.f && p.E <= kRouterThreads) {
        // a single token with plain top-k: the whole CTA selects, then groups directly
        __shared__ float s_tops[kMaxTopK];
        topk_one_token_cta(p.sel, p.score, p.E, p.k, p.scaling, p.topk_idx, p.topk_w, s_idx, s_tops,
                           reinterpret_cast<unsigned long long *>(sm_run),
                           reinterpret_cast<unsigned long long *>(sm_off), tid);
        if (p.do_group)
            group_one_token(s_idx, p.E, p.k, p.counts, p.offsets, p.perm, p.unique, p.n_unique, p.slots, tid);
        return;
    }
    for (int t = warp; t < nt; t += kRouterThreads / 32)
        topk_token(p.sel + (size_t)(t0 + t) * p.E, p.score + (size_t)(t0 + t) * p.E, p.E, p.k, p.scaling, p.top_p,
                   p.topk_idx + (size_t)(t0 + t) * p.k, p.topk_w + (size_t)(t0 + t) * p.k, s_idx + t * p.k);
    if (!p.do_group) return;
    __syncthreads();
    if (gridDim.y == 1) {
        // one token tile: group straight from this CTA's top-k
        if (p.slots)
            group_block<kRouterThreads, 0>(s_idx, p.T * p.k, p.E, p.counts, p.offsets, p.perm, p.unique,
                                           p.n_unique, p.slots, sm_run, sm_off, p.status, tid);
        else if (warp == 0)
            group_warp(s_idx, true, p.T * p.k, p.E, p.counts, p.offsets, p.perm, p.unique, p.n_unique, sm_run, sm_off,
                       p.status, p.slots);
        return;
    }
    // the last token tile runs the grouping, from a shared-memory copy of all tiles' top-k
    // when it fits in this CTA's x buffers (one parallel pass instead of dependent loads)
    if (tid == 0) s_flag = atom_inc_acq_rel(p.group_counter, gridDim.y - 1) == gridDim.y - 1;
    __syncthreads();
    if (!s_flag) return;
    const int n = p.T * p.k;
    const size_t dyn = p.do_gemv ? (size_t)p.x_bufs * p.x_rows * p.H * 2 : 0;
    const bool in_smem = (size_t)n * 4 <= dyn;
    if (in_smem) {
        int *s_all = reinterpret_cast<int *>(r_smem);
        for (int a = tid; a < n; a += kRouterThreads) s_all[a] = __ldcg(p.topk_idx + a);
        __syncthreads();
    }
    if (warp == 0)
        group_warp(in_smem ? reinterpret_cast<const int32_t *>(r_smem) : p.topk_idx, in_smem, n, p.E, p.counts,
                   p.offsets, p.perm, p.unique, p.n_unique, sm_run, sm_off, p.status, p.slots);
}

// ---------------------------------------------------------------------------- batches
// Grouping of n assignments by the eight warps of a CTA (the larger batches): warp w
// counts its contiguous segment of assignment ids per expert, one exclusive scan over
// (expert, warp) gives every warp its first position inside each expert's bucket, and
// each warp then places its segment in ascending a.  Same results as group_warp.
// cnt: shared memory [8][E]; idx: the n top-k indices (shared or global memory).
__device__ void group_warps8(const int32_t *idx, bool src_smem, int n, int E, int32_t *counts, int32_t *offsets,
                             int32_t *perm, int32_t *unique, int32_t *n_unique, int4 *slots, int *cnt, int *status)
{
    constexpr int kW = kRouterThreads / 32;
    __shared__ int s_wsum[kW], s_wnz[kW];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < kW * E; i += kRouterThreads) cnt[i] = 0;
    __syncthreads();
    const int seg = (n + kW - 1) / kW;
    const int a0 = min(n, warp * seg), a1 = min(n, a0 + seg);
    int *my = cnt + warp * E;
    for (int base = a0; base < a1; base += 32) {
        const int a = base + lane;
        int e = (a < a1) ? (src_smem ? idx[a] : __ldcg(idx + a)) : -1;
        if (a < a1 && (e < -1 || e >= E)) {   // -1: dropped by top-p, no expert
            record_error(status, MOE_ERR_DEVICE_BOUNDS);
            e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // exclusive scan over experts: thread t owns experts [t*P, t*P + P)
    const int P = (E + kRouterThreads - 1) / kRouterThreads;
    const int e0 = tid * P;
    int local = 0, nz = 0;
    for (int i = 0; i < P; ++i) {
        const int e = e0 + i;
        if (e < E) {
            int c = 0;
#pragma unroll
            for (int w = 0; w < kW; ++w) c += cnt[w * E + e];
            local += c;
            nz += c > 0;
        }
    }
    int incl = local, incl_nz = nz;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        const int u = __shfl_up_sync(0xffffffffu, incl_nz, off);
        if (lane >= off) {
            incl += v;
            incl_nz += u;
        }
    }
    if (lane == 31) {
        s_wsum[warp] = incl;
        s_wnz[warp] = incl_nz;
    }
    __syncthreads();
    int pre = 0, pre_nz = 0;
    for (int w = 0; w < warp; ++w) {
        pre += s_wsum[w];
        pre_nz += s_wnz[w];
    }
    int run = pre + incl - local, ur = pre_nz + incl_nz - nz;
    for (int i = 0; i < P; ++i) {
        const int e = e0 + i;
        if (e < E) {
            int c = 0;
#pragma unroll
            for (int w = 0; w < kW; ++w) {
                const int cw = cnt[w * E + e];
                cnt[w * E + e] = run + c;   // warp w's first position in bucket e
                c += cw;
            }
            counts[e] = c;
            offsets[e] = run;
            if (c > 0) {
                if (slots) slots[ur] = make_int4(e, c, run, 0);
                unique[ur++] = e;
            }
            run += c;
        }
    }
    if (tid == kRouterThreads - 1) {
        offsets[E] = run;
        *n_unique = ur;
    }
    __syncthreads();
    for (int base = a0; base < a1; base += 32) {
        const int a = base + lane;
        int e = (a < a1) ? (src_smem ? idx[a] : __ldcg(idx + a)) : -1;
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) perm[my[e] + __popc(peers & ((1u << lane) - 1u))] = a;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
        __syncwarp();
    }
}

// Router for batches of more than one token tile: CTA (expert tile, token tile) forms the
// 16 x 32 block of logits as an fp32 GEMM tile.  K passes through a four-stage ring of
// shared memory in chunks of 128, filled by every thread with 16-byte asynchronous copies
// (coalesced rows; small rows make many bulk-copy requests, which the copy engine serves
// too slowly here); rows are padded so that the lanes' loads meet no bank conflicts.
// Warp w takes k in [16w, 16w + 16) of every chunk; lane (tg, eg) accumulates
// tokens {tg, tg + 8} x experts
// {eg + 4i}; the eight warps' partial sums are added in warp order (deterministic).
// Scores, top-k and grouping then follow as in the GEMV router.  For the int8 expert
// path every CTA also tracks the |x| maxima of its rows and, after the GEMM, writes its
// share of x's limb blocks; for the int4 mma path the CTAs of expert tile 0 write x in
// B-fragment order from the chunks they stage.
constexpr int kRtE = 32;                        // experts per CTA
constexpr int kRtK = 128;                       // K per stage
constexpr int kRtWStride = kRtK + 4;            // fp32 router row stride in shared memory
constexpr int kRtXStride = kRtK + 8;            // fp16 token row stride
constexpr int kRtStageBytes = kRtE * kRtWStride * 4 + kRouterTokTile * kRtXStride * 2;
constexpr int kRtStages = 4;
constexpr int kRtSmem = kRtStages * kRtStageBytes;
static_assert(kRouterTokTile <= 32, "one token row per lane of the issuing warp");
static_assert(kRtSmem >= kRouterThreads / 32 * kRouterTokTile * (kRtE + 1) * 4, "partial sums alias the ring");

__global__ void __launch_bounds__(kRouterThreads) router_tile_kernel(RouterParams p)
{
    extern __shared__ __align__(16) unsigned char r_smem[];
    __shared__ float s_amax[kRouterTokTile];
    __shared__ int s_flag;
    __shared__ int s_idx[kRouterTokTile * kMaxTopK];

    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tt = blockIdx.y, t0 = tt * kRouterTokTile, nt = min(kRouterTokTile, p.T - t0);
    const int eb = blockIdx.x * kRtE, ne = min(kRtE, p.E - eb);
    if (tt == 0) {
        // the expert tile's router rows into L2 while earlier work drains
        for (int r = 0; r < ne; ++r) {
            const char *row = reinterpret_cast<const char *>(p.w + (size_t)(eb + r) * p.H);
            for (int o = tid * 128; o < p.H * 4; o += kRouterThreads * 128)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(row + o));
        }
    }
    pdl_wait();

    const int nch = (p.H + kRtK - 1) / kRtK;
    auto stage_w = [&](int s) { return reinterpret_cast<float *>(r_smem + (size_t)s * kRtStageBytes); };
    auto stage_x = [&](int s) {
        return reinterpret_cast<uint16_t *>(r_smem + (size_t)s * kRtStageBytes + kRtE * kRtWStride * 4);
    };
    auto issue = [&](int c) {   // all threads: chunk c into stage c % kRtStages (one commit group)
        if (c < nch) {
            const int s = c % kRtStages, k0 = c * kRtK, kc = min(kRtK, p.H - k0);
            constexpr int kW16 = kRtK / 4, kX16 = kRtK / 8;   // 16-byte pieces of a row
            for (int j = tid; j < kRtE * kW16; j += kRouterThreads) {
                const int r = j / kW16, q = j % kW16;
                if (r < ne && 4 * q < kc)
                    cp_async16(stage_w(s) + r * kRtWStride + 4 * q, p.w + (size_t)(eb + r) * p.H + k0 + 4 * q);
            }
            for (int j = tid; j < kRouterTokTile * kX16; j += kRouterThreads) {
                const int r = j / kX16, q = j % kX16;
                if (r < nt && 8 * q < kc)
                    cp_async16(stage_x(s) + r * kRtXStride + 8 * q, p.x + (size_t)(t0 + r) * p.H + k0 + 8 * q);
            }
        }
        cp_async_commit();
    };
    for (int c = 0; c < kRtStages - 1; ++c) issue(c);

    const bool conv = p.x_limbs != nullptr;
    const bool perm = blockIdx.x == 0 && p.x_perm != nullptr;
    const int nblk = (p.H + kLimbBlockK - 1) / kLimbBlockK;

    const int tg = lane & 7, eg = lane >> 3;
    float acc[2][8];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[a][i] = 0.f;
    // |x| maxima of tokens tg and tg + 8 over this warp's k (for the limbs' row scales)
    __half2 amx[2] = {__float2half2_rn(0.f), __float2half2_rn(0.f)};
    for (int c = 0; c < nch; ++c) {
        const int s = c % kRtStages, kc = min(kRtK, p.H - c * kRtK);
        cp_async_wait<kRtStages - 2>();   // this thread's pieces of chunk c have landed
        __syncthreads();                  // everyone's have; stage (c - 1) % S is free again
        issue(c + kRtStages - 1);
        const float *ws = stage_w(s);
        const uint16_t *xs = stage_x(s);
        if (perm) {
            for (int j = tid; j < nt * (kRtK / 8); j += kRouterThreads) {
                const int r = j / (kRtK / 8), k8 = (j % (kRtK / 8)) * 8;
                if (k8 < kc) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(xs + r * kRtXStride + k8);
                    *reinterpret_cast<uint4 *>(p.x_perm + (size_t)(t0 + r) * p.H + c * kRtK + k8) =
                        make_uint4(pack_lo(v.x, v.z), pack_hi(v.x, v.z), pack_lo(v.y, v.w), pack_hi(v.y, v.w));
                }
            }
        }
        const int kw0 = warp * (kRtK / 8), kw1 = min(kc, kw0 + kRtK / 8);
        for (int k = kw0; k < kw1; k += 4) {
            float xf[2][4];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const uint2 xr = *reinterpret_cast<const uint2 *>(xs + (tg + 8 * a) * kRtXStride + k);
                if (conv)
                    amx[a] = __hmax2(amx[a], __hmax2(__habs2(*reinterpret_cast<const __half2 *>(&xr.x)),
                                                     __habs2(*reinterpret_cast<const __half2 *>(&xr.y))));
                const float2 lo = __half22float2(*reinterpret_cast<const __half2 *>(&xr.x));
                const float2 hi = __half22float2(*reinterpret_cast<const __half2 *>(&xr.y));
                xf[a][0] = lo.x;
                xf[a][1] = lo.y;
                xf[a][2] = hi.x;
                xf[a][3] = hi.y;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 wv = *reinterpret_cast<const float4 *>(ws + (eg + 4 * i) * kRtWStride + k);
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    acc[a][i] = fmaf(wv.x, xf[a][0], acc[a][i]);
                    acc[a][i] = fmaf(wv.y, xf[a][1], acc[a][i]);
                    acc[a][i] = fmaf(wv.z, xf[a][2], acc[a][i]);
                    acc[a][i] = fmaf(wv.w, xf[a][3], acc[a][i]);
                }
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    // partial sums [warp][token][expert] over the (now idle) ring, then summed in warp order
    float *red = reinterpret_cast<float *>(r_smem);
    float *amx_w = red + (kRouterThreads / 32) * kRouterTokTile * kRtE;   // [warp][token]
#pragma unroll
    for (int a = 0; a < 2; ++a) {
#pragma unroll
        for (int i = 0; i < 8; ++i) red[(warp * kRouterTokTile + tg + 8 * a) * kRtE + eg + 4 * i] = acc[a][i];
        if (conv && eg == 0)
            amx_w[warp * kRouterTokTile + tg + 8 * a] =
                fmaxf(__low2float(amx[a]), __high2float(amx[a]));
    }
    __syncthreads();
    if (conv) {
        // x as int8 limbs: this CTA writes limb blocks b = blockIdx.x (mod expert tiles) of
        // the tile's rows (x read again, from L2)
        if (tid < nt) {
            float m = 0.f;
#pragma unroll
            for (int w = 0; w < kRouterThreads / 32; ++w) m = fmaxf(m, amx_w[w * kRouterTokTile + tid]);
            s_amax[tid] = m;
            if (blockIdx.x == 0) p.x_limb_scale[t0 + tid] = pow2f(-limb_shift(m));
        }
        __syncthreads();
        for (int b = blockIdx.x; b < nblk; b += gridDim.x)
            for (int j = tid; j < nt * (kLimbBlockK / 8); j += kRouterThreads) {
                const int r = j / (kLimbBlockK / 8), k8 = (j % (kLimbBlockK / 8)) * 8, k = b * kLimbBlockK + k8;
                const uint4 v = k < p.H ? __ldcg(reinterpret_cast<const uint4 *>(p.x + (size_t)(t0 + r) * p.H + k))
                                        : make_uint4(0u, 0u, 0u, 0u);
                limb_encode8(v, pow2f(limb_shift(s_amax[r])), p.x_limbs + ((size_t)(t0 + r) * nblk + b) * kLimbBlockBytes,
                             k8);
            }
    }
    for (int o = tid; o < kRouterTokTile * kRtE; o += kRouterThreads) {
        const int t = o / kRtE, e = o % kRtE;
        if (t < nt && e < ne) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kRouterThreads / 32; ++w) v += red[w * kRouterTokTile * kRtE + o];
            const size_t g = (size_t)(t0 + t) * p.E + eb + e;
            const float sc = sigmoid_ref(v);
            p.logits[g] = v;
            p.score[g] = sc;
            p.sel[g] = sc + p.bias[eb + e];
        }
    }
    // the last expert tile of this token tile runs its top-k
    __syncthreads();
    if (tid == 0) s_flag = atom_inc_acq_rel(p.tile_counters + tt, gridDim.x - 1) == gridDim.x - 1;
    __syncthreads();
    if (!s_flag) return;
    for (int t = warp; t < nt; t += kRouterThreads / 32)
        topk_token(p.sel + (size_t)(t0 + t) * p.E, p.score + (size_t)(t0 + t) * p.E, p.E, p.k, p.scaling, p.top_p,
                   p.topk_idx + (size_t)(t0 + t) * p.k, p.topk_w + (size_t)(t0 + t) * p.k, s_idx + t * p.k);
    if (!p.do_group) return;
    // the last token tile groups the whole batch
    __syncthreads();
    if (tid == 0) s_flag = atom_inc_acq_rel(p.group_counter, gridDim.y - 1) == gridDim.y - 1;
    __syncthreads();
    if (!s_flag) return;
    const int n = p.T * p.k;
    int *cnt = reinterpret_cast<int *>(r_smem);
    int *s_all = cnt + (kRouterThreads / 32) * p.E;
    const bool in_smem = (size_t)((kRouterThreads / 32) * p.E + n) * 4 <= (size_t)kRtSmem;
    if (in_smem) {
        for (int a = tid; a < n; a += kRouterThreads) s_all[a] = __ldcg(p.topk_idx + a);
        __syncthreads();
    }
    group_warps8(in_smem ? s_all : p.topk_idx, in_smem, n, p.E, p.counts, p.offsets, p.perm, p.unique, p.n_unique,
                 p.slots, cnt, p.status);
}

__global__ void __launch_bounds__(kRouterThreads) group_kernel(GroupParams p)
{
    extern __shared__ int g_cnt[];   // [8][E]
    group_warps8(p.topk_idx, false, p.T * p.k, p.E, p.counts, p.offsets, p.perm, p.unique, p.n_unique, nullptr,
                 g_cnt, p.status);
}

__global__ void __launch_bounds__(256) combine_kernel(CombineParams p)
{
    pdl_trigger();   // a router launched behind this kernel may start (it waits for it)
    pdl_wait();      // y_assign and y_shared come from the down kernel (no-op without PDL)
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)p.T * p.H) return;
    const int t = static_cast<int>(i / p.H), m = static_cast<int>(i % p.H);
    float acc = p.n_shared ? p.y_shared[i] : 0.f;
    for (int j = 0; j < p.k; ++j) {
        const float w = p.topk_w[(size_t)t * p.k + j];
        if (w != 0.f) acc = fmaf(w, p.y_assign[((size_t)t * p.k + j) * p.H + m], acc);   // 0: dropped by top-p
    }
    p.y[i] = __half_as_ushort(__float2half_rn(acc));
}

// x of a host-buffer call: page-locked host memory mapped into the device's address space
// -> the workspace's staging buffer, as the first kernel of the layer's launch chain.  Each
// thread reads its (up to four) 16-byte pieces over the bus first (uncached: the host
// rewrites the buffer between calls), while the previous layer is still running, and
// writes them only once that layer is complete (it is the buffer's last reader), so the
// bus round trip overlaps the previous layer and the router behind keeps its early start.
__global__ void __launch_bounds__(256) host_x_kernel(const uint4 *src, uint4 *dst, size_t n16)
{
    pdl_trigger();   // the router launched behind this kernel may start (it waits for it)
    const size_t base = (size_t)blockIdx.x * (256 * 4) + threadIdx.x;
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const size_t i = base + (size_t)j * 256;
        if (i < n16)
            asm volatile("ld.global.cv.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v[j].x), "=r"(v[j].y), "=r"(v[j].z), "=r"(v[j].w)
                         : "l"(src + i));
    }
    pdl_wait();      // the previous layer no longer reads the staging buffer
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const size_t i = base + (size_t)j * 256;
        if (i < n16) dst[i] = v[j];
    }
}

// x -> int8 limbs on its own (the staged expert entry point, which runs no router):
// one CTA per token row
__global__ void __launch_bounds__(kRouterThreads) x_limbs_kernel(const uint16_t *x, int H, unsigned char *limbs,
                                                                 float *scale)
{
    __shared__ float red_max[kRouterThreads / 32];
    const int t = blockIdx.x, tid = threadIdx.x;
    const uint16_t *row = x + (size_t)t * H;
    float m = 0.f;
    for (int k8 = 8 * tid; k8 < H; k8 += 8 * kRouterThreads)
        m = fmaxf(m, amax8(__ldg(reinterpret_cast<const uint4 *>(row + k8))));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((tid & 31) == 0) red_max[tid >> 5] = m;
    __syncthreads();
    m = 0.f;
#pragma unroll
    for (int w = 0; w < kRouterThreads / 32; ++w) m = fmaxf(m, red_max[w]);
    const int sh = limb_shift(m);
    const int nblk = (H + kLimbBlockK - 1) / kLimbBlockK;
    unsigned char *dst = limbs + (size_t)t * nblk * kLimbBlockBytes;
    for (int k8 = 8 * tid; k8 < nblk * kLimbBlockK; k8 += 8 * kRouterThreads) {
        const uint4 v = k8 < H ? __ldg(reinterpret_cast<const uint4 *>(row + k8)) : make_uint4(0u, 0u, 0u, 0u);
        limb_encode8(v, pow2f(sh), dst + (size_t)(k8 / kLimbBlockK) * kLimbBlockBytes, k8 % kLimbBlockK);
    }
    if (tid == 0) scale[t] = pow2f(-sh);
}

cudaError_t launch_x_limbs(const uint16_t *x, int T, int H, unsigned char *limbs, float *scale, cudaStream_t s)
{
    if (T <= 0) return cudaSuccess;
    x_limbs_kernel<<<T, kRouterThreads, 0, s>>>(x, H, limbs, scale);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------- static scratch
// Scratch of moe_route_static, which allocates nothing: the router's token-tile
// counters, then score, selection score and logits for kStaticRouteElems (token,
// expert) pairs.  Zero at module load; the counters are brought back to zero by every
// complete call (atomicInc wraps), the float arrays are written before they are read.
static __device__ __align__(256) unsigned char g_route_scratch[kStaticRouteBytes];

// The array's device address belongs to the CUDA context that loaded this module: a
// context created later (after cudaDeviceReset, or a driver-API context of the caller)
// has its own copy at another address.  The address is therefore cached per context,
// keyed by the context's process-unique id (cuCtxGetId), never by device ordinal.
namespace {
struct CtxFns {
    PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    PFN_cuCtxGetId_v12000 get_id = nullptr;
    bool ok = false;
};

const CtxFns &ctx_fns()
{
    static CtxFns f = [] {
        CtxFns r;
        cudaDriverEntryPointQueryResult q;
        void *a = nullptr, *b = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            r.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(a);
            r.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(b);
            r.ok = true;
        }
        return r;
    }();
    return f;
}
}  // namespace

cudaError_t static_route_scratch(void **ptr)
{
    static std::mutex mu;
    static unsigned long long ids[kStaticRouteContexts] = {};
    static void *addr[kStaticRouteContexts] = {};
    static int next = 0;
    const CtxFns &f = ctx_fns();
    if (!f.ok) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (f.get_current(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
    if (!ctx) {
        // no context is current on this thread yet: the runtime call creates (and makes
        // current) the device's primary context, whose id is taken below
        void *a = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&a, g_route_scratch);
        if (e != cudaSuccess) return e;
        if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorUnknown;
    }
    unsigned long long id = 0;
    if (f.get_id(ctx, &id) != CUDA_SUCCESS) return cudaErrorUnknown;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kStaticRouteContexts; ++i)
        if (addr[i] && ids[i] == id) {
            *ptr = addr[i];
            return cudaSuccess;
        }
    void *a = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&a, g_route_scratch);
    if (e != cudaSuccess) return e;
    ids[next] = id;   // the oldest entry gives way when every slot is taken
    addr[next] = a;
    next = (next + 1) % kStaticRouteContexts;
    *ptr = a;
    return cudaSuccess;
}

// ---------------------------------------------------------------------------- launchers
// Shared-memory limits and carveout of the small kernels (once per process and device:
// the attributes belong to the kernels).  The carveout asks for the largest shared
// memory split so that the expert kernels' CTAs can start beside the router's.
cudaError_t router_prepare()
{
    cudaError_t e = cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRouterMaxDynSmem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(router_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(x_limbs_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(router_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRtSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(router_tile_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return e;
}

cudaError_t launch_router(const RouterParams &p0, bool pdl, cudaStream_t s)
{
    RouterParams p = p0;
    // more than one token tile: the GEMM-tiled router
    const bool tiled = p.do_gemv && p.T > kRouterTokTile;
    const int gx = tiled ? (p.E + kRtE - 1) / kRtE : p.do_gemv ? p.E : 1;
    const int gy = (p.T + kRouterTokTile - 1) / kRouterTokTile;
    size_t smem = tiled ? (size_t)kRtSmem : 0;
    if (p.do_gemv && !tiled) {
        const size_t row = (size_t)p.H * 2;
        p.x_rows = std::min(p.T, kRouterXRows);
        p.x_bufs = (p.T > p.x_rows && 2 * p.x_rows * row <= (size_t)kRouterMaxDynSmem) ? 2 : 1;
        smem = (size_t)p.x_bufs * p.x_rows * row;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gx, gy);
    cfg.blockDim = dim3(kRouterThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return tiled ? cudaLaunchKernelEx(&cfg, router_tile_kernel, p) : cudaLaunchKernelEx(&cfg, router_kernel, p);
}

cudaError_t launch_group(const GroupParams &p, cudaStream_t s)
{
    group_kernel<<<1, kRouterThreads, (size_t)(kRouterThreads / 32) * p.E * sizeof(int), s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_host_x(const void *src, void *dst, size_t bytes, cudaStream_t s)
{
    const size_t n16 = bytes / 16;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n16 + 1023) / 1024));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, host_x_kernel, static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), n16);
}

cudaError_t launch_combine(const CombineParams &p, bool pdl, cudaStream_t s)
{
    const size_t n = (size_t)p.T * p.H;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, combine_kernel, p);
}

}  // namespace moe
