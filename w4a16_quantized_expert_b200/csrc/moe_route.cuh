// moe_route.cuh -- routing pieces shared by the router kernels (moe_router.cu) and the
// fused decode-layer kernel (moe_fused.cu): the reference sigmoid, the top-k of one token
// (and the adaptive expert top-p) and the grouping of one token tile.
//
// DeepSeek-V3-style sigmoid router ("Show HN: 低速のコンピュータでGLM 5.2を動かす方法",
// section 実装済み機能): s = sigmoid(logit) evaluated in fp64 and rounded to fp32; selection
// score s + bias in fp32; the k best (ties -> lower expert index); weights
// scaling * s_j / sum s.  Grouping: the batch MoE union of the same page, in a fixed order.
#pragma once

#include <cuda_fp16.h>
#include <math.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

// barrier of the NT threads that run a grouping (BAR 0: the whole CTA)
template <int NT, int BAR>
__device__ __forceinline__ void group_sync()
{
    if constexpr (BAR == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

__device__ __forceinline__ float sigmoid_ref(float logit)
{
    return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(logit))));
}

// order-preserving map of a float to an unsigned key (larger float -> larger key)
__device__ __forceinline__ unsigned float_key(float v)
{
    const unsigned b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// ---------------------------------------------------------------------------- top-k
// One warp per token: k rounds, each one warp-wide max of the selection keys and one
// min of the expert indices holding that max (equal scores -> lower expert index).
template <int kPer>
__device__ void topk_token_t(const float *sel_row, const float *score_row, int E, int k, float scaling,
                             float top_p, int32_t *idx_out, float *w_out, int *idx_smem)
{
    const int lane = threadIdx.x & 31;
    // selection keys and the unbiased scores, loaded together (one round trip)
    unsigned key[kPer];
    float sco[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        const bool in = e < E;
        key[i] = in ? float_key(__ldcg(sel_row + e)) : 0u;
        sco[i] = in ? __ldcg(score_row + e) : 0.f;
    }
    uint32_t taken = 0;
    int my_idx = 0;
    float my_score = 0.f;
    for (int j = 0; j < k; ++j) {
        // this lane's best remaining expert (its score travels with it)
        unsigned bk = 0u, be = 0xffffffffu;
        float bs = 0.f;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !(taken >> i & 1u) && (be == 0xffffffffu || key[i] > bk)) {
                bk = key[i];
                be = (unsigned)e;
                bs = sco[i];
            }
        }
        const unsigned kmax = __reduce_max_sync(0xffffffffu, bk);
        const unsigned win = __reduce_min_sync(0xffffffffu, (be != 0xffffffffu && bk == kmax) ? be : 0xffffffffu);
        const float ws = __shfl_sync(0xffffffffu, bs, (int)(win & 31u));
        if ((int)(win & 31u) == lane) taken |= 1u << (win >> 5);
        if (lane == j) {
            my_idx = (int)win;
            my_score = ws;
        }
    }
    // combine weights from the unbiased scores, summed in order j = 0..k-1
    double s_mine = 0.0;
    if (lane < k) s_mine = static_cast<double>(my_score);
    double sum = 0.0;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, s_mine, j);
    if (top_p > 0.f) {
        // adaptive expert top-p: rank of this lane's expert among the k by score (equal
        // scores: lower expert index first); the score mass ranked ahead of it, summed in
        // rank order; kept while that mass is below top_p of the k's mass
        int rank = 0;
        for (int i = 0; i < k; ++i) {
            const float si = __shfl_sync(0xffffffffu, my_score, i);
            const int ei = __shfl_sync(0xffffffffu, my_idx, i);
            if (lane < k && (si > my_score || (si == my_score && ei < my_idx))) ++rank;
        }
        double before = 0.0;
        for (int r = 0; r < k; ++r) {
            const unsigned who = __ballot_sync(0xffffffffu, lane < k && rank == r);
            const double v = __shfl_sync(0xffffffffu, s_mine, __ffs(who) - 1);
            if (r < rank) before += v;
        }
        const bool keep = lane < k && before < static_cast<double>(top_p) * sum;
        const unsigned kept = __ballot_sync(0xffffffffu, keep);
        // kept experts first, in top-k order, weights renormalised over them
        double sum2 = 0.0;
        for (int j = 0; j < k; ++j) {
            const double v = __shfl_sync(0xffffffffu, s_mine, j);
            if (kept >> j & 1u) sum2 += v;
        }
        const int pos = __popc(kept & ((1u << lane) - 1u)), m = __popc(kept);
        if (keep) {
            idx_smem[pos] = my_idx;
            idx_out[pos] = my_idx;
            w_out[pos] = static_cast<float>(static_cast<double>(scaling) * (s_mine / sum2));
        }
        __syncwarp();
        if (lane < k && lane >= m) {
            idx_smem[lane] = -1;
            idx_out[lane] = -1;
            w_out[lane] = 0.f;
        }
        return;
    }
    if (lane < k) {
        idx_smem[lane] = my_idx;
        idx_out[lane] = my_idx;
        w_out[lane] = static_cast<float>(static_cast<double>(scaling) * (s_mine / sum));
    }
}

__device__ __forceinline__ void topk_token(const float *sel_row, const float *score_row, int E, int k, float scaling,
                           float top_p, int32_t *idx_out, float *w_out, int *idx_smem)
{
    if (E <= 256) topk_token_t<8>(sel_row, score_row, E, k, scaling, top_p, idx_out, w_out, idx_smem);
    else topk_token_t<kMaxExperts / 32>(sel_row, score_row, E, k, scaling, top_p, idx_out, w_out, idx_smem);
}

// counts and offsets of all E experts from the slot list group_block leaves in its scratch
// (by binary search): the part of the grouping nothing downstream of the fused kernel's
// routing flag waits for.
template <int NT>
__device__ void group_counts(int nu, int nk, int E, int32_t *counts, int32_t *offsets, const int *sm_a,
                             const int *sm_b, int tid, int ns = kRouterTokTile * kMaxTopK)
{
    const int *s_uniq = sm_a + ns;
    const int *s_uoff = sm_b, *s_ucnt = sm_b + ns;
    for (int e = tid; e < E; e += NT) {
        int lo = 0, hi = nu;   // first slot whose expert is >= e
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (s_uniq[mid] < e) lo = mid + 1;
            else hi = mid;
        }
        const bool has = lo < nu && s_uniq[lo] == e;
        counts[e] = has ? s_ucnt[lo] : 0;
        offsets[e] = lo < nu ? s_uoff[lo] : nk;
    }
}

// Grouping of a single token tile by the whole top-k CTA (n = T*k <= 512 assignments):
// every assignment's rank in (expert, a) order is counted directly from the n keys in
// shared memory, which gives perm; the first assignment of each expert places that
// expert's slot (expert, count, offset); counts and offsets of all E experts follow by
// binary search in the slot list.  Same results as group_warp.  NT threads (thread index
// tid) take part and meet at barrier BAR (0: the whole CTA).  The scratch sm_a and sm_b
// hold 2 ns ints each (ns >= n).
template <int NT, int BAR, bool kCounts = true>
__device__ int2 group_block(const int *s_idx, int n, int E, int32_t *counts, int32_t *offsets, int32_t *perm,
                            int32_t *unique, int32_t *n_unique, int4 *slots, int *sm_a, int *sm_b, int *status,
                            int tid, int ns = kRouterTokTile * kMaxTopK)
{
    constexpr int kPer = kRouterTokTile * kMaxTopK / NT;   // assignments per thread
    int *s_first = sm_a, *s_uniq = sm_a + ns;
    int *s_uoff = sm_b, *s_ucnt = sm_b + ns;
    __shared__ int s_nu;
    int rk[kPer], ee[kPer], lt[kPer], eq[kPer];
    bool fi[kPer];
    int nk = 0;   // assignments that reach an expert (top-p drops are -1)
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int a = tid + u * NT;
        fi[u] = false;
        if (u == 0)
            for (int b = 0; b < n; ++b) nk += s_idx[b] >= 0;
        if (a < n && s_idx[a] >= 0) {
            const int e = s_idx[a];
            if (e >= E) record_error(status, MOE_ERR_DEVICE_BOUNDS);
            int l = 0, q = 0, qb = 0;
            for (int b = 0; b < n; ++b) {
                const int e2 = s_idx[b];
                l += (e2 >= 0) & (e2 < e);
                q += e2 == e;
                qb += (e2 == e) & (b < a);
            }
            rk[u] = l + qb;
            ee[u] = e;
            lt[u] = l;
            eq[u] = q;
            fi[u] = qb == 0;
            perm[rk[u]] = a;
            s_first[rk[u]] = fi[u] ? 1 : 0;
        }
    }
    group_sync<NT, BAR>();
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        if (fi[u]) {
            int si = 0;
            for (int r = 0; r < rk[u]; ++r) si += s_first[r];
            slots[si] = make_int4(ee[u], eq[u], lt[u], 0);
            unique[si] = ee[u];
            s_uniq[si] = ee[u];
            s_uoff[si] = lt[u];
            s_ucnt[si] = eq[u];
            if (lt[u] + eq[u] == nk) s_nu = si + 1;   // the last expert's slot
        }
    }
    group_sync<NT, BAR>();
    const int nu = s_nu;
    if (tid == 0) {
        *n_unique = nu;
        offsets[E] = nk;
    }
    if constexpr (kCounts) group_counts<NT>(nu, nk, E, counts, offsets, sm_a, sm_b, tid, ns);
    return make_int2(nu, nk);
}

}  // namespace moe
