// moe_fused.cu -- the decode-sized MoE layer (T <= 16 tokens) in one persistent launch:
// router GEMV, sigmoid scores, top-k, grouping, gate/up, SiLU * up, down and the combine
// with the shared expert, with no grid-wide barrier between the steps.
//
// Sources: MoE routing fused into small-batch custom kernels ("GLM-5.3-Flash 320B MoEを
// 4枚のCMP 170HXで動かすvLLMレシピ", section "Ampere世代のGPU向けに最適化された独自カーネル群");
// the DeepSeek-V3-style sigmoid router, int4 with per-row scales, the shared expert and the
// batch MoE union ("Show HN: 低速のコンピュータでGLM 5.2を動かす方法", section 実装済み機能);
// NVFP4 decoded in registers inside the matmul ("GTX 1070向け35BパラメータMoEモデル推論
// エンジン公開", section "VRAMとシステムメモリで重みを分割する設計"); one replayed unit per
// decode step (same page, section "Pascal世代の制約をCUDAグラフとカーネル最適化で克服").
//
// Why one launch.  A decode layer streams about ten experts' weights once.  As separate
// kernels (router, gate/up, down, combine) every step pays a launch, a pipeline fill and a
// drain, and no routed expert's weights can stream before the whole router grid is done.
// Here one grid of two CTAs per SM walks one ordered list of work items:
//   router tasks   expert e's logits for the T tokens (its fp32 router row times each x
//                  row, summed in the same order as the router kernel, so the logits are
//                  the same bits), the sigmoid and selection scores; tasks e < ceil(H/256)
//                  also write x's int8 limbs (int4 weights).  The task that completes the
//                  set runs the top-k and the grouping and publishes them.
//   gate/up items  the shared expert first (it needs no routing), then the routed experts
//                  in ascending order; an item is (expert, 64 output rows, <= 8 tokens).
//   down items     the shared expert, then the routed ones, likewise.
// CTA b's first item is item b; later ones are claimed from a counter, so items start in
// list order.  A CTA has a producer warp (TMA ring of weight boxes, bulk copies of the B
// rows) and four consumer warps (the inner loops of the per-step expert kernel).
// Dependencies are flags carrying the call's epoch, never grid barriers:
//   * the B rows of a gate/up item (x limbs) wait for the x-limb flag; routed items wait
//     for the routing flag, after which the producer builds its slot table;
//   * the B rows of a down item (h limbs, or h for NVFP4) wait for their token chunk's
//     flag, set by the CTA whose gate/up item completed the chunk (after converting the
//     chunk's h rows to limbs);
//   * the combine of a 64-row output tile runs in the CTA whose down item completed it.
// Weights never wait: the producer issues the weight boxes of an item's first stages
// before it waits for the item's B rows.  Items are claimed in dependency order and no
// completion step waits on anything, so the oldest unfinished item always has its inputs;
// every wait is bounded all the same (a timeout is recorded, never a hang).
#include <cuda_fp16.h>
#include <math.h>

#include "moe_device.cuh"
#include "moe_expert.cuh"
#include "moe_internal.h"
#include "moe_route.cuh"

namespace moe {

constexpr int kFuRows = kConsumerWarps * kRowTile;   // 64 output rows per item
constexpr int kFuTok = 8;                           // tokens per item
constexpr int kFuJc = 6;                            // router-row float4 per virtual thread per pass
constexpr int kFuVirt = 8;                          // router: virtual warps (256 virtual threads)
constexpr int kFuRMax = 1;                          // experts per router task at most
constexpr int kFuCT = kConsumerWarps * 32;          // consumer threads
constexpr int kFuHdr = 48;                          // header words of the slot table (see FuTable)
constexpr int kFuSeen = 16;                         // first header word of the seen-flag bits
constexpr int kFuSlotsMax = 32;                     // ring slots at most (mbarrier pairs)
constexpr int kFuIssue = 4;                         // slots the producer warp fills at once (a lane each)

enum { kCtlEpoch = 0, kCtlRoute = 1, kCtlXl = 2, kCtlRouter = 3, kCtlWork = 4, kCtlDone = 5, kCtlXlDone = 6 };

// The ring is made of slots, each one 64-row x 128-byte weight box (256 K values; and for
// NVFP4 its E4M3 scale box) plus one K block of the item's B rows.  A gate/up stage takes
// two consecutive slots (g with the B rows, then u), a down stage one: both kinds of item
// keep the same number of weight bytes in flight.
template <int FMT>
struct FuCfg {
    static constexpr bool kNv = FMT == MOE_FMT_NVFP4;
    static constexpr bool kLimbs = !kNv;
    static constexpr int kScales = kNv ? kConsumerWarps * kScaleBoxSmem : 0;   // 64 rows x 16 scale bytes
    static constexpr int kBRow = kNv ? 2 * kLimbBlockK + 16 : kLimbBlockBytes;  // one token, one K block
    static constexpr int kBLen = kNv ? 2 * kLimbBlockK : kLimbBlockBytes;       // bytes copied per row
    static constexpr int kBOff = kMatStage + kScales;                           // B rows inside a slot
};

// shared memory of a CTA besides the ring: zero row, top-k of the batch and grouping scratch
// (ns = T k assignments), router sums, slot table of `cap` experts, header, barriers
template <int FMT>
__host__ __device__ constexpr size_t fu_fixed_smem(int cap, int ns)
{
    return 1024 + FuCfg<FMT>::kBRow + (size_t)5 * ns * 4 +
           (size_t)(kFuRMax * kFuVirt * kFusedMaxT + kFusedMaxT) * 4 + (size_t)5 * (cap + 2) * 4 + kFuHdr * 4 +
           (2 * kFuSlotsMax + 1 + 2 * kItemQ) * 8 + 64;
}

// ------------------------------------------------------------------ flags
__device__ __forceinline__ unsigned *ctl_word(const FusedParams &p, int w) { return p.ctl + w * kSyncLine; }
__device__ __forceinline__ unsigned *chunk_flag(const FusedParams &p, int c) { return p.chunk_flag + c * kSyncLine; }
__device__ __forceinline__ unsigned *chunk_ctr(const FusedParams &p, int c) { return p.chunk_ctr + c * kSyncLine; }
__device__ __forceinline__ unsigned *tile_ctr(const FusedParams &p, int t) { return p.tile_ctr + t * kSyncLine; }

__device__ __forceinline__ unsigned ld_relaxed(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// after a relaxed load saw a released value: acquire its writes, for this thread's generic
// loads and for the bulk copies it issues next (async proxy)
__device__ __forceinline__ void acquire_seen()
{
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void st_release(unsigned *p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait until *flag == want, then acquire.  Gives up after kWaitTimeoutNs, recording
// MOE_ERR_DEVICE_TIMEOUT.  The flag is written by another CTA of this grid.  Polls are
// relaxed loads spaced by a short sleep (hundreds of warps may poll one flag); the acquire
// fence comes once, when the value is seen.
__device__ __forceinline__ bool wait_flag(const unsigned *flag, unsigned want, int *status)
{
    if (ld_relaxed(flag) != want) {
        const unsigned long long t0 = globaltimer_ns();
        for (unsigned long long it = 1;; ++it) {
            __nanosleep(128);
            if (ld_relaxed(flag) == want) break;
            if (it >= kWaitMaxIters || ((it & 15) == 0 && globaltimer_ns() - t0 > kWaitTimeoutNs)) {
                record_error(status, MOE_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
    acquire_seen();
    return true;
}

// ------------------------------------------------------------------ work items
struct FuItem {
    int kind;    // 0 router task, 1 gate/up, 2 down, 3 x-limb task
    int e;       // expert (-1: shared); router task: its expert
    int row0;    // first output row
    int tok0;    // first bucket position of the token chunk
    int ntok;    // tokens (1..8)
    int boff;    // bucket start in perm order (0 for the shared expert)
    int K;       // input dimension
    int chunk;   // index of the chunk's counter and flag: boff + tok0, or T*k + tok0 (shared)
};

// slot table in shared memory: the non-empty routed experts in ascending order
struct FuTable {
    int *e, *cnt, *off, *bgu, *bdn;   // expert, tokens, bucket start, first gate/up / down item
    int *hdr;   // [0] slots, [1] total items, [2] abort, [3] consumer fail, [4..7] item queue,
                // [8] first shared down item, [9] first routed down item, [10] down items per tile,
                // [16..33] one bit per token chunk whose flag this CTA has already seen
};

__device__ __forceinline__ int fu_chunks(int n) { return (n + kFuTok - 1) / kFuTok; }

// Item list: [0, NX) x-limb tasks, [NX, NH) router tasks, [NH, A1) shared gate/up, then
// routed gate/up, shared down, routed down (boundaries of the last three in the table).
__device__ __forceinline__ FuItem fu_decode(const FusedParams &p, const FuTable &tb, int i, int NX, int NH, int A1)
{
    FuItem it = {};
    if (i < NX) {
        it.kind = 3;
        it.e = i;   // the limb block
        return it;
    }
    if (i < NH) {
        it.kind = 0;
        it.e = i - NX;
        return it;
    }
    if (i < A1) {   // shared gate/up
        const int local = i - NH, tiles = p.I_sh / kFuRows;
        it.kind = 1;
        it.e = -1;
        it.row0 = (local % tiles) * kFuRows;
        it.tok0 = (local / tiles) * kFuTok;
        it.ntok = min(kFuTok, p.T - it.tok0);
        it.K = p.H;
        it.chunk = p.T * p.k + it.tok0;
        return it;
    }
    const int A2 = tb.hdr[8], A3 = tb.hdr[9];
    if (i >= A2 && i < A3) {   // shared down
        const int local = i - A2, tiles = p.H / kFuRows;
        it.kind = 2;
        it.e = -1;
        it.row0 = (local % tiles) * kFuRows;
        it.tok0 = (local / tiles) * kFuTok;
        it.ntok = min(kFuTok, p.T - it.tok0);
        it.K = p.I_sh;
        it.chunk = p.T * p.k + it.tok0;
        return it;
    }
    const bool gu = i < A2;
    const int *base = gu ? tb.bgu : tb.bdn;
    const int local0 = i - (gu ? A1 : A3);
    int lo = 0, hi = tb.hdr[0] - 1;   // last slot whose first item is <= local0
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (base[mid] <= local0) lo = mid;
        else hi = mid - 1;
    }
    const int local = local0 - base[lo], tiles = (gu ? p.I : p.H) / kFuRows;
    it.kind = gu ? 1 : 2;
    it.e = tb.e[lo];
    it.row0 = (local % tiles) * kFuRows;
    it.tok0 = (local / tiles) * kFuTok;
    it.ntok = min(kFuTok, tb.cnt[lo] - it.tok0);
    it.boff = tb.off[lo];
    it.K = gu ? p.H : p.I;
    it.chunk = it.boff + it.tok0;
    return it;
}

// The producer warp's slot table from the router's compact slot list (after the routing
// flag): per slot its first gate/up and down item, the list boundaries and the number of
// down items that cover each output row tile.
__device__ void fu_build_table(const FusedParams &p, const FuTable &tb, int cap, int A1)
{
    const int lane = threadIdx.x & 31;
    // the count and the first 32 slots in one round trip (slots past the count are unused)
    const int4 s_first = lane < cap ? __ldcg(p.slots + lane) : make_int4(0, 0, 0, 0);
    int nu = __ldcg(p.n_unique);
    if (nu < 0 || nu > cap) {
        if (lane == 0) record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
        nu = nu < 0 ? 0 : cap;
    }
    const int tg = p.I / kFuRows, td = p.H / kFuRows;
    int acc_g = 0, acc_d = 0, acc_c = 0;
    for (int b = 0; b < nu; b += 32) {
        const int j = b + lane;
        int e = 0, cnt = 0, off = 0;
        if (j < nu) {
            const int4 s = b == 0 ? s_first : __ldcg(p.slots + j);
            e = s.x;
            cnt = s.y;
            off = s.z;
            if (e < 0 || e >= p.E || cnt < 0 || off < 0 || off + cnt > p.T * p.k) {
                record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                e = 0;
                cnt = 0;
                off = 0;
            }
        }
        const int nc = fu_chunks(cnt);
        int ig = tg * nc, id = td * nc, ic = nc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int vg = __shfl_up_sync(0xffffffffu, ig, o), vd = __shfl_up_sync(0xffffffffu, id, o),
                      vc = __shfl_up_sync(0xffffffffu, ic, o);
            if (lane >= o) {
                ig += vg;
                id += vd;
                ic += vc;
            }
        }
        if (j < nu) {
            tb.e[j] = e;
            tb.cnt[j] = cnt;
            tb.off[j] = off;
            tb.bgu[j] = acc_g + ig - tg * nc;
            tb.bdn[j] = acc_d + id - td * nc;
        }
        acc_g += __shfl_sync(0xffffffffu, ig, 31);
        acc_d += __shfl_sync(0xffffffffu, id, 31);
        acc_c += __shfl_sync(0xffffffffu, ic, 31);
    }
    if (lane == 0) {
        const int nsh = p.n_shared ? fu_chunks(p.T) : 0;
        tb.bgu[nu] = acc_g;
        tb.bdn[nu] = acc_d;
        tb.hdr[0] = nu;
        tb.hdr[8] = A1 + acc_g;
        tb.hdr[9] = A1 + acc_g + nsh * td;
        tb.hdr[1] = tb.hdr[9] + acc_d;
        tb.hdr[10] = nsh + acc_c;
    }
    __syncwarp();
}

// B row of token j of an item (its K block 0; block b lies kBLen * b bytes further):
// x limbs / x (gate/up) or h limbs / h (down); NULL for a bad routing index.
template <int FMT>
__device__ __forceinline__ const unsigned char *fu_brow(const FusedParams &p, const FuItem &it, int j)
{
    constexpr bool kLimbs = FuCfg<FMT>::kLimbs;
    const bool sh = it.e < 0;
    const int bpos = it.tok0 + j;
    auto lrow = [](int K) { return (size_t)((K + kLimbBlockK - 1) / kLimbBlockK) * kLimbBlockBytes; };
    if (it.kind == 1) {
        int t = bpos;
        if (!sh) {
            const int a = __ldcg(p.perm + it.boff + bpos);
            t = (a >= 0 && a < p.T * p.k) ? a / p.k : -1;
            if (t < 0) {
                record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                return nullptr;
            }
        }
        return kLimbs ? p.x_limbs + (size_t)t * lrow(p.H) : reinterpret_cast<const unsigned char *>(p.x + (size_t)t * p.H);
    }
    if (kLimbs)
        return sh ? p.hsh_limbs + (size_t)bpos * lrow(p.I_sh) : p.h_limbs + (size_t)(it.boff + bpos) * lrow(p.I);
    return sh ? reinterpret_cast<const unsigned char *>(p.h_sh + (size_t)bpos * p.I_sh)
              : reinterpret_cast<const unsigned char *>(p.h + (size_t)(it.boff + bpos) * p.I);
}

// ------------------------------------------------------------------ completion steps
// A completion counter increment whose result is looked at later (the atomic's round trip
// is then hidden behind the next item's stages): kind 1, a gate/up row tile of a token
// chunk (the CTA that completes the chunk converts its h rows and sets the chunk's flag);
// kind 2, a down item of an output row tile (the CTA that completes the tile combines it).
struct FuPend {
    int kind;
    unsigned old, target;
    unsigned *ctr;
    int sh, tok0, ntok, boff, chunk, row0;
};

template <int FMT>
__device__ void fu_settle(const FusedParams &p, FuPend &pd, int ltid, unsigned epoch)
{
    if (pd.kind == 0) return;   // uniform over the consumer threads
    __shared__ int s_go;
    if (ltid == 0) s_go = pd.old == pd.target;
    consumer_sync();
    if (s_go) {
        if (pd.kind == 1) {
            if constexpr (FuCfg<FMT>::kLimbs) {
                auto lrow = [](int K) { return (size_t)((K + kLimbBlockK - 1) / kLimbBlockK) * kLimbBlockBytes; };
                if (pd.sh)
                    convert_h_rows<kFuCT, 1>(p.h_sh + (size_t)pd.tok0 * p.I_sh, p.I_sh,
                                             p.hsh_limbs + (size_t)pd.tok0 * lrow(p.I_sh), p.hsh_limb_scale + pd.tok0,
                                             p.h_amax + p.T * p.k + pd.tok0, pd.ntok, p.I_sh, ltid);
                else
                    convert_h_rows<kFuCT, 1>(p.h + (size_t)(pd.boff + pd.tok0) * p.I, p.I,
                                             p.h_limbs + (size_t)(pd.boff + pd.tok0) * lrow(p.I),
                                             p.h_limb_scale + pd.boff + pd.tok0, p.h_amax + pd.boff + pd.tok0, pd.ntok,
                                             p.I, ltid);
            }
            if (ltid == 0) st_release(chunk_flag(p, pd.chunk), epoch);
        } else {
            // combine of output rows [row0, row0 + 64) of every token: shared + sum_j w_j y_j
            // in fp32, in the order shared, j = 0 .. k-1 (weight 0: dropped by top-p)
            // (the weights and rows of 8 experts at a time are loaded together; a dropped
            // entry's row is loaded but not used)
            for (int o = ltid; o < p.T * kFuRows; o += kFuCT) {
                const int t = o / kFuRows, m = pd.row0 + o % kFuRows;
                const size_t i = (size_t)t * p.H + m;
                float acc = p.n_shared ? __ldcg(p.y_shared + i) : 0.f;
                for (int j0 = 0; j0 < p.k; j0 += 8) {
                    float w[8], v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const bool in = j0 + j < p.k;
                        w[j] = in ? __ldcg(p.topk_w + (size_t)t * p.k + j0 + j) : 0.f;
                        v[j] = in ? __ldcg(p.y_assign + ((size_t)t * p.k + j0 + j) * p.H + m) : 0.f;
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (w[j] != 0.f) acc = fmaf(w[j], v[j], acc);
                }
                p.y[i] = __half_as_ushort(__float2half_rn(acc));
            }
        }
    }
    consumer_sync();   // s_go is rewritten by the next settle
    pd.kind = 0;
}

// The completion counts run two items behind: pq[0] is a finished item not counted yet,
// pq[1] one whose count went out after the item that followed it (its atomic's release
// then finds the item's stores long done, and its result is looked at one item later
// still).  `now`: count pq[0] and look at the result at once (before a down item that
// may wait for this CTA's own chunk conversion, and at the end).
template <int FMT>
__device__ void fu_advance(const FusedParams &p, FuPend (&pq)[2], int ltid, unsigned epoch, bool now)
{
    fu_settle<FMT>(p, pq[1], ltid, epoch);
    if (pq[0].kind) {
        consumer_sync();   // every thread's stores of the item precede its count
        if (ltid == 0) pq[0].old = atom_inc_acq_rel(pq[0].ctr, pq[0].target);
        pq[1] = pq[0];
        pq[0].kind = 0;
        if (now) fu_settle<FMT>(p, pq[1], ltid, epoch);
    }
}

// ------------------------------------------------------------------ router and x-limb tasks
// The logits of experts [r R, r R + R) for the T tokens.  128 consumer threads stand in
// for the router kernel's 256 (thread t carries virtual threads t and t + 128) so that
// every logit is summed in exactly the router kernel's order: per virtual thread an fma
// chain over its float4 of the router row, a butterfly inside each (virtual) warp, the
// eight warp sums in order.  The x values of two tokens are loaded before their products.
__device__ void fu_router_task(const FusedParams &p, int r, int R, int ltid, float (*red)[kFusedMaxT])
{
    const int lane = ltid & 31, rw = ltid >> 5;
    const int T = p.T, H4 = p.H >> 2;
    for (int q = 0; q < R; ++q) {
        const int e = r * R + q;
        if (e >= p.E) break;
        float acc[2][kFusedMaxT];
#pragma unroll
        for (int v = 0; v < 2; ++v)
#pragma unroll
            for (int t = 0; t < kFusedMaxT; ++t) acc[v][t] = 0.f;
        const float4 *wrow = reinterpret_cast<const float4 *>(p.wt.router_w + (size_t)e * p.H);
        for (int jc = 0; jc < 16 && jc * 256 < H4; jc += kFuJc) {
            float4 wv[2][kFuJc];
#pragma unroll
            for (int v = 0; v < 2; ++v)
#pragma unroll
                for (int jj = 0; jj < kFuJc; ++jj) {
                    const int h4 = (jc + jj) * 256 + ltid + 128 * v;
                    wv[v][jj] = (jc + jj < 16 && h4 < H4) ? __ldg(wrow + h4) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
            for (int t0 = 0; t0 < kFusedMaxT; t0 += 2) {
                if (t0 < T) {
                    uint2 xr[2][2][kFuJc];
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                        for (int v = 0; v < 2; ++v)
#pragma unroll
                            for (int jj = 0; jj < kFuJc; ++jj) {
                                const int h4 = (jc + jj) * 256 + ltid + 128 * v;
                                xr[tt][v][jj] = (t0 + tt < T && jc + jj < 16 && h4 < H4)
                                                    ? __ldcg(reinterpret_cast<const uint2 *>(p.x + (size_t)(t0 + tt) * p.H) + h4)
                                                    : make_uint2(0u, 0u);
                            }
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        if (t0 + tt < T) {
#pragma unroll
                            for (int v = 0; v < 2; ++v)
#pragma unroll
                                for (int jj = 0; jj < kFuJc; ++jj) {
                                    const int h4 = (jc + jj) * 256 + ltid + 128 * v;
                                    if (jc + jj < 16 && h4 < H4) {
                                        const float2 xa = __half22float2(*reinterpret_cast<const __half2 *>(&xr[tt][v][jj].x));
                                        const float2 xb = __half22float2(*reinterpret_cast<const __half2 *>(&xr[tt][v][jj].y));
                                        float &a = acc[v][t0 + tt];
                                        a = fmaf(wv[v][jj].x, xa.x, a);
                                        a = fmaf(wv[v][jj].y, xa.y, a);
                                        a = fmaf(wv[v][jj].z, xb.x, a);
                                        a = fmaf(wv[v][jj].w, xb.y, a);
                                    }
                                }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < kFusedMaxT; ++t) {
            if (t < T) {
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    float s = acc[v][t];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                    if (lane == 0) red[q * kFuVirt + rw + 4 * v][t] = s;
                }
            }
        }
    }
    consumer_sync();
    for (int o = ltid; o < R * T; o += kFuCT) {
        const int q = o / T, t = o % T, e = r * R + q;
        if (e >= p.E) continue;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kFuVirt; ++w) v += red[q * kFuVirt + w][t];
        const size_t i = (size_t)t * p.E + e;
        const float sc = static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(v))));
        p.logits[i] = v;
        p.score[i] = sc;
        p.sel[i] = sc + p.wt.router_bias[e];
    }
    consumer_sync();   // red is rewritten by the next task
}

// Limb block b (K values [256 b, 256 b + 256)) of every x row, for the int8 tensor path:
// the rows' largest magnitudes (over all of H; the loads of two rows go out together), then
// the block's three int8 limbs per value (the representation the router kernel writes);
// block 0's task also writes the rows' scales.
__device__ void fu_xlimb_task(const FusedParams &p, int b, int ltid, float (*red)[kFusedMaxT], float *s_amax)
{
    const int lane = ltid & 31, rw = ltid >> 5;
    const int T = p.T, H8 = p.H >> 3;
    float m[kFusedMaxT];
#pragma unroll
    for (int t = 0; t < kFusedMaxT; ++t) m[t] = 0.f;
#pragma unroll
    for (int t0 = 0; t0 < kFusedMaxT; t0 += 2) {
        if (t0 < T) {
            for (int j0 = 0; j0 < H8; j0 += 8 * kFuCT) {
                uint4 v[2][8];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        const int j = j0 + jj * kFuCT + ltid;
                        v[tt][jj] = (t0 + tt < T && j < H8)
                                        ? __ldcg(reinterpret_cast<const uint4 *>(p.x + (size_t)(t0 + tt) * p.H) + j)
                                        : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) m[t0 + tt] = fmaxf(m[t0 + tt], amax8(v[tt][jj]));
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kFusedMaxT; ++t) {
        if (t < T) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m[t] = fmaxf(m[t], __shfl_xor_sync(0xffffffffu, m[t], off));
            if (lane == 0) red[rw][t] = m[t];
        }
    }
    consumer_sync();
    if (ltid < T) s_amax[ltid] = fmaxf(fmaxf(red[0][ltid], red[1][ltid]), fmaxf(red[2][ltid], red[3][ltid]));
    consumer_sync();
    const size_t lrow = (size_t)((p.H + kLimbBlockK - 1) / kLimbBlockK) * kLimbBlockBytes;
    for (int j0 = 0; j0 < T * 32; j0 += 2 * kFuCT) {
        uint4 v[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = j0 + u * kFuCT + ltid, r = j >> 5, k = b * kLimbBlockK + (j & 31) * 8;
            v[u] = (j < T * 32 && k < p.H) ? __ldcg(reinterpret_cast<const uint4 *>(p.x + (size_t)r * p.H + k))
                                           : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = j0 + u * kFuCT + ltid, r = j >> 5, k8 = (j & 31) * 8;
            if (j < T * 32)
                limb_encode8(v[u], pow2f(limb_shift(s_amax[r])),
                             p.x_limbs + (size_t)r * lrow + (size_t)b * kLimbBlockBytes, k8);
        }
    }
    if (b == 0 && ltid < T) p.x_limb_scale[ltid] = pow2f(-limb_shift(s_amax[ltid]));
    consumer_sync();   // red / s_amax are rewritten by the next task
}

// The task that completes the router set: the top-k of every token (a warp per token) and
// the grouping (the four consumer warps), published with the routing flag; the counts and
// offsets of every expert after it.
template <int FMT>
__device__ void fu_route_finish(const FusedParams &p, int ltid, unsigned epoch, int *s_idx, int *grp_a, int *grp_b)
{
    const int rw = ltid >> 5, ns = p.T * p.k;
    for (int t = rw; t < p.T; t += kConsumerWarps)
        topk_token(p.sel + (size_t)t * p.E, p.score + (size_t)t * p.E, p.E, p.k, p.scaling, p.top_p,
                   p.topk_idx + (size_t)t * p.k, p.topk_w + (size_t)t * p.k, s_idx + t * p.k);
    consumer_sync();
    const int2 nn = group_block<kFuCT, 1, false>(s_idx, ns, p.E, p.counts, p.offsets, p.perm, p.unique,
                                                 p.n_unique, p.slots, grp_a, grp_b, p.status, ltid, ns);
    consumer_sync();
    if (ltid == 0) st_release(ctl_word(p, kCtlRoute), epoch);
    // counts and offsets of every expert: results of the call, but nothing in it waits for them
    group_counts<kFuCT>(nn.x, nn.y, p.E, p.counts, p.offsets, grp_a, grp_b, ltid, ns);
}

// ------------------------------------------------------------------ inner loops
// int4 codes of one chunk pair (64 K values) of the warp's 16 rows as s8 bytes 16 x code,
// against the B limbs (int8 tensor path); a0 / a1: the weight boxes of g and u (gate/up) or
// of d (down, a1 unused).  Accumulation is exact in s32, in two chains (even / odd elements).
template <bool GU, int NN>
__device__ __forceinline__ void fu_pair_limbs(uint32_t a0, uint32_t a1, const Lane &L, int q, const uint4 (&Bq)[NN],
                                              int (&acc)[2][GU ? 2 : 1][NN][4])
{
    constexpr int M = GU ? 2 : 1;
    uint32_t ev[M][4], od[M][4];
#pragma unroll
    for (int m = 0; m < M; ++m) {
        uint32_t r[4];
        ldmatrix_x4(r[0], r[1], r[2], r[3], (m ? a1 : a0) + L.off[q]);
#pragma unroll
        for (int i = 0; i < 4; ++i) int4_word_to_s8x16(r[i], ev[m][i], od[m][i]);
    }
#pragma unroll
    for (int n = 0; n < NN; ++n) {
        const uint4 B = Bq[n];
#pragma unroll
        for (int m = 0; m < M; ++m) {
            mma_s8(acc[0][m][n], ev[m][0], ev[m][1], ev[m][2], ev[m][3], B.x, B.y);
            mma_s8(acc[1][m][n], od[m][0], od[m][1], od[m][2], od[m][3], B.z, B.w);
        }
    }
}

// NVFP4 codes of one chunk pair of the warp's 16 rows times their E4M3 block scales, decoded
// to fp16 in registers, against fp16 B values (X0, X1: this lane's 16 bytes of the two
// chunks), f16 mma with fp32 accumulation.  a[m]: weight box, sc[m]: the box's scale bytes.
template <int M>
__device__ __forceinline__ void fu_pair_nv(const uint32_t (&a)[M], const unsigned char *const (&sc)[M], const Lane &L,
                                           int q, const uint4 &X0, const uint4 &X1, float (&acc)[M][4])
{
    uint32_t A[M][2][2][4];   // [mat][chunk][row g / g + 8][pairs]
#pragma unroll
    for (int m = 0; m < M; ++m) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(r0, r1, r2, r3, a[m] + L.off[q]);
        const unsigned char *s = sc[m] + L.bx * kScaleBoxSmem;
        const int b0 = 4 * q + (L.tq >> 1);   // block of (chunk 2q, word tq)
        dequant_nvfp4_word(r0, e4m3_to_half2(s[L.g * kScaleBoxBytes + b0]), A[m][0][0]);
        dequant_nvfp4_word(r1, e4m3_to_half2(s[(L.g + 8) * kScaleBoxBytes + b0]), A[m][0][1]);
        dequant_nvfp4_word(r2, e4m3_to_half2(s[L.g * kScaleBoxBytes + b0 + 2]), A[m][1][0]);
        dequant_nvfp4_word(r3, e4m3_to_half2(s[(L.g + 8) * kScaleBoxBytes + b0 + 2]), A[m][1][1]);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const uint4 X = c == 0 ? X0 : X1;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            mma_16816(acc[m], A[m][c][0][0], A[m][c][1][0], A[m][c][0][1], A[m][c][1][1], X.x, X.y);
            mma_16816(acc[m], A[m][c][0][2], A[m][c][1][2], A[m][c][0][3], A[m][c][1][3], X.z, X.w);
        }
    }
}

// the ring position of the consumers (or the producer): slot and its phase
struct FuRing {
    int slot;
    uint32_t phase;
    __device__ __forceinline__ void next(int S)
    {
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

// ------------------------------------------------------------------ expert items
// Consumer side of a gate/up or down item on the int8 tensor path (int4 weights).  NN = 1
// for items of 1-2 tokens (B columns (limb, token) = (g / 2, g % 2)), NN = 3 otherwise
// (n-tile = limb, column = token).  The epilogue forms sum(code * X) = S0 + 256 S1 +
// 65536 S2 exactly in 64-bit integers and scales it in fp64; gate/up stores h in fp16 and
// gathers the rows' largest |h|; down stores y_assign (y_shared).
template <bool GU, int NN>
__device__ __forceinline__ bool fu_consume_limbs(const FusedParams &p, const FuItem &it, unsigned char *ring,
                                                 uint64_t *full, uint64_t *empty, FuRing &rg, const Lane &L,
                                                 uint32_t zsm, FuPend (&pq)[2], volatile int *cfail,
                                                 volatile int *abort_flag, const FuTable &tb, unsigned epoch)
{
    using Cf = FuCfg<MOE_FMT_INT4_ROWSCALE>;
    constexpr int M = GU ? 2 : 1;
    const int S = p.stages, SB = p.stage_bytes;
    const bool sh = it.e < 0;
    const int nkb = (it.K + kLimbBlockK - 1) / kLimbBlockK;
    const int lcol = NN == 1 ? (L.g >> 1) : 0;
    const int tcol = NN == 1 ? (L.g & 1) : L.g;
    const bool bval = lcol < 3 && tcol < it.ntok;
    const uint32_t boffs = (uint32_t)(Cf::kBOff + tcol * Cf::kBRow + lcol * kLimbBlockK + 16 * L.tq);
    const int ltid = threadIdx.x;

    const int rows_all = GU ? (sh ? p.I_sh : p.I) : p.H;
    const int ez = sh ? 0 : it.e;
    const int rowA = it.row0 + L.rw * kRowTile + L.g;
    const float *sc0 = GU ? (sh ? p.wt.sh_g_scale : p.wt.g_scale) : (sh ? p.wt.sh_d_scale : p.wt.d_scale);
    const float *sc1 = sh ? p.wt.sh_u_scale : p.wt.u_scale;
    float rs0[2], rs1[2] = {0.f, 0.f}, xsc[2] = {0.f, 0.f};
    int asg[2] = {0, 0};
    bool uval[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        rs0[h] = __ldg(sc0 + (size_t)ez * rows_all + rowA + 8 * h);
        if (GU) rs1[h] = __ldg(sc1 + (size_t)ez * rows_all + rowA + 8 * h);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int t = NN == 1 ? u : 2 * L.tq + u;
        uval[u] = (NN == 1 ? L.tq == 0 : true) && t < it.ntok;
    }

    int acc2[2][M][NN][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
            for (int n = 0; n < NN; ++n)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc2[h][m][n][c] = 0;

    bool ok = true;
    for (int s = 0; s < nkb; ++s) {
        // the stage's slots: g (with the B rows) and u, or d (with the B rows)
        const int s0 = rg.slot;
        if (!mbar_wait(&full[rg.slot], rg.phase, p.status)) { ok = false; break; }
        rg.next(S);
        int s1 = s0;
        if (GU) {
            s1 = rg.slot;
            if (!mbar_wait(&full[rg.slot], rg.phase, p.status)) { ok = false; break; }
            rg.next(S);
        }
        if (s == 0) {
            // the activation scales and assignment ids of the lane's tokens (published before
            // this item's B rows were copied)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (!uval[u]) continue;
                const int t = NN == 1 ? u : 2 * L.tq + u;
                const int bpos = it.tok0 + t;
                asg[u] = sh ? bpos : __ldcg(p.perm + it.boff + bpos);
                if (GU) {
                    const int tok = sh ? bpos : ((asg[u] >= 0 && asg[u] < p.T * p.k) ? asg[u] / p.k : -1);
                    if (tok >= 0) xsc[u] = __ldcg(p.x_limb_scale + tok);
                } else {
                    xsc[u] = __ldcg(sh ? p.hsh_limb_scale + bpos : p.h_limb_scale + it.boff + bpos);
                }
            }
        }
        const int npairs = min(4, (it.K - s * kLimbBlockK) / 64);   // K is a multiple of 64
        const uint32_t base0 = smem_u32(ring + (size_t)s0 * SB), base1 = smem_u32(ring + (size_t)s1 * SB);
        const uint32_t bb = bval ? base0 + boffs : zsm + 16 * L.tq;
        uint4 B[4][NN];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int n = 0; n < NN; ++n) B[q][n] = lds128(bb + n * kLimbBlockK + 64 * q);
        const uint32_t a0 = base0 + L.bx * kBoxSmem, a1 = base1 + L.bx * kBoxSmem;
        if (npairs == 4) {
#pragma unroll
            for (int q = 0; q < 4; ++q) fu_pair_limbs<GU, NN>(a0, a1, L, q, B[q], acc2);
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (q < npairs) fu_pair_limbs<GU, NN>(a0, a1, L, q, B[q], acc2);
        }
        __syncwarp();
        if (L.lane == 0) {
            mbar_arrive(&empty[s0]);
            if (GU) mbar_arrive(&empty[s1]);
        }
    }
    if (!ok) {
        *cfail = 1;
        *abort_flag = 1;
    }
    // the previous item's completion step (its atomic has long returned), then agreement
    // on failure
    fu_advance<MOE_FMT_INT4_ROWSCALE>(p, pq, ltid, epoch, false);
    consumer_sync();
    if (*cfail) return false;

    int acc[M][NN][4];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int n = 0; n < NN; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[m][n][c] = acc2[0][m][n][c] + acc2[1][m][n][c];
    float hmax[2] = {0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        long long Sv[M];
        if constexpr (NN == 1) {
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const int v0 = acc[m][0][c] >> 4;
                const int v1 = __shfl_down_sync(0xffffffffu, v0, 1);
                const int v2 = __shfl_down_sync(0xffffffffu, v0, 2);
                Sv[m] = (long long)v0 + 256ll * v1 + 65536ll * v2;
            }
        } else {
#pragma unroll
            for (int m = 0; m < M; ++m)
                Sv[m] = (long long)(acc[m][0][c] >> 4) + 256ll * (acc[m][1][c] >> 4) + 65536ll * (acc[m][2][c] >> 4);
        }
        const int u = c & 1, h = c >> 1;
        if (!uval[u]) continue;
        const int row = rowA + 8 * h;
        const int bpos = it.tok0 + (NN == 1 ? u : 2 * L.tq + u);
        if (GU) {
            const double xs = (double)xsc[u];
            const float gv = (float)((double)Sv[0] * xs * (double)rs0[h]);
            const float uv = (float)((double)Sv[M - 1] * xs * (double)rs1[h]);
            const float hv = gv / (1.f + expf(-gv)) * uv;
            __half *dst = sh ? p.h_sh + (size_t)bpos * p.I_sh : p.h + (size_t)(it.boff + bpos) * p.I;
            const __half hh = __float2half_rn(hv);
            dst[row] = hh;
            hmax[u] = fmaxf(hmax[u], fabsf(__half2float(hh)));
        } else {
            const float yv = (float)((double)Sv[0] * (double)xsc[u] * (double)rs0[h]);
            if (sh) {
                p.y_shared[(size_t)bpos * p.H + row] = yv;
            } else {
                const int a = asg[u];
                if (a >= 0 && a < p.T * p.k) p.y_assign[(size_t)a * p.H + row] = yv;
                else record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
            }
        }
    }
    if (GU) {
        if (!sh) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int a = asg[u];
                if (uval[u] && (a < 0 || a >= p.T * p.k)) record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
            }
        }
        // the h rows' largest magnitudes (per token: lanes of a quad-column, then one atomic)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float m = hmax[u];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const int t = NN == 1 ? u : 2 * L.tq + u;
            if (L.g == 0 && (NN == 1 ? L.tq == 0 : true) && t < it.ntok)
                atomicMax(p.h_amax + (sh ? p.T * p.k : it.boff) + it.tok0 + t, __float_as_uint(m));
        }
    }
    // count this item (gate/up: a row tile of its token chunk; down: one of its output row
    // tile's items); the completing CTA converts or combines, one item later
    // this item's count (gate/up: a row tile of its token chunk; down: one of its output
    // row tile's items) goes out after the next item's stages
    FuPend &pd = pq[0];
    pd.sh = sh;
    pd.tok0 = it.tok0;
    pd.ntok = it.ntok;
    pd.boff = it.boff;
    pd.chunk = it.chunk;
    pd.row0 = it.row0;
    if (GU) {
        pd.kind = 1;
        pd.target = (unsigned)(rows_all / kFuRows) - 1u;
        pd.ctr = chunk_ctr(p, it.chunk);
    } else {
        pd.kind = 2;
        pd.target = (unsigned)tb.hdr[10] - 1u;
        pd.ctr = tile_ctr(p, it.row0 / kFuRows);
    }
    return true;
}

// NVFP4 items: E2M1 codes times the E4M3 block scale decoded to fp16 in registers, fp16
// B rows (x or h) from shared memory, f16 mma with fp32 accumulation, tensor scale in the
// epilogue.  One n-tile of up to 8 tokens.
template <bool GU>
__device__ __forceinline__ bool fu_consume_nv(const FusedParams &p, const FuItem &it, unsigned char *ring,
                                              uint64_t *full, uint64_t *empty, FuRing &rg, const Lane &L,
                                              uint32_t zsm, FuPend (&pq)[2], volatile int *cfail,
                                              volatile int *abort_flag, const FuTable &tb, unsigned epoch)
{
    using Cf = FuCfg<MOE_FMT_NVFP4>;
    constexpr int M = GU ? 2 : 1;
    const int S = p.stages, SB = p.stage_bytes;
    const bool sh = it.e < 0;
    const int nkb = it.K / kLimbBlockK;   // NVFP4: K is a multiple of 256
    const int ltid = threadIdx.x;
    float part[M][4];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) part[m][c] = 0.f;
    bool ok = true;
    for (int s = 0; s < nkb; ++s) {
        const int s0 = rg.slot;
        if (!mbar_wait(&full[rg.slot], rg.phase, p.status)) { ok = false; break; }
        rg.next(S);
        int s1 = s0;
        if (GU) {
            s1 = rg.slot;
            if (!mbar_wait(&full[rg.slot], rg.phase, p.status)) { ok = false; break; }
            rg.next(S);
        }
        unsigned char *st0 = ring + (size_t)s0 * SB, *st1 = ring + (size_t)s1 * SB;
        const uint32_t bsm = (L.g < it.ntok ? smem_u32(st0 + Cf::kBOff + L.g * Cf::kBRow) : zsm) + 16 * L.tq;
        uint32_t a[M];
        const unsigned char *sc[M];
        a[0] = smem_u32(st0) + L.bx * kBoxSmem;
        sc[0] = st0 + kMatStage;
        if (GU) {
            a[M - 1] = smem_u32(st1) + L.bx * kBoxSmem;
            sc[M - 1] = st1 + kMatStage;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
            fu_pair_nv<M>(a, sc, L, q, lds128(bsm + 128 * q), lds128(bsm + 128 * q + 64), part);
        __syncwarp();
        if (L.lane == 0) {
            mbar_arrive(&empty[s0]);
            if (GU) mbar_arrive(&empty[s1]);
        }
    }
    if (!ok) {
        *cfail = 1;
        *abort_flag = 1;
    }
    fu_advance<MOE_FMT_NVFP4>(p, pq, ltid, epoch, false);
    consumer_sync();
    if (*cfail) return false;

    const int rows_all = GU ? (sh ? p.I_sh : p.I) : p.H;
    const float *sc0 = GU ? (sh ? p.wt.sh_g_scale : p.wt.g_scale) : (sh ? p.wt.sh_d_scale : p.wt.d_scale);
    const float *sc1 = sh ? p.wt.sh_u_scale : p.wt.u_scale;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int col = 2 * L.tq + (c & 1);
        if (col >= it.ntok) continue;
        const int row = it.row0 + L.rw * kRowTile + L.g + (c >> 1) * 8;
        const int bpos = it.tok0 + col;
        if (GU) {
            const float gv = part[0][c] * mat_scale<MOE_FMT_NVFP4>(sc0, it.e, rows_all, row);
            const float uv = part[M - 1][c] * mat_scale<MOE_FMT_NVFP4>(sc1, it.e, rows_all, row);
            const float hv = gv / (1.f + expf(-gv)) * uv;
            __half *dst = sh ? p.h_sh + (size_t)bpos * p.I_sh : p.h + (size_t)(it.boff + bpos) * p.I;
            dst[row] = __float2half_rn(hv);
        } else {
            const float yv = part[0][c] * mat_scale<MOE_FMT_NVFP4>(sc0, it.e, rows_all, row);
            if (sh) {
                p.y_shared[(size_t)bpos * p.H + row] = yv;
            } else {
                const int a = __ldcg(p.perm + it.boff + bpos);
                if (a >= 0 && a < p.T * p.k) p.y_assign[(size_t)a * p.H + row] = yv;
                else record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
            }
        }
    }
    // this item's count (gate/up: a row tile of its token chunk; down: one of its output
    // row tile's items) goes out after the next item's stages
    FuPend &pd = pq[0];
    pd.sh = sh;
    pd.tok0 = it.tok0;
    pd.ntok = it.ntok;
    pd.boff = it.boff;
    pd.chunk = it.chunk;
    pd.row0 = it.row0;
    if (GU) {
        pd.kind = 1;
        pd.target = (unsigned)(rows_all / kFuRows) - 1u;
        pd.ctr = chunk_ctr(p, it.chunk);
    } else {
        pd.kind = 2;
        pd.target = (unsigned)tb.hdr[10] - 1u;
        pd.ctr = tile_ctr(p, it.row0 / kFuRows);
    }
    return true;
}

// ------------------------------------------------------------------ the kernel
template <int FMT>
__global__ void __launch_bounds__(kFfnThreads, 2) fused_kernel(const __grid_constant__ LayerMaps maps,
                                                               const FusedParams p)
{
    using Cf = FuCfg<FMT>;
    const int S = p.stages, SB = p.stage_bytes;   // ring slots and bytes per slot
    const int ns = p.T * p.k;                      // assignments of the batch
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *ring =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *zrow_sm = ring + (size_t)S * SB;
    int *s_idx = reinterpret_cast<int *>(zrow_sm + Cf::kBRow);   // [T k] the batch's top-k
    int *grp_a = s_idx + ns;                                      // grouping scratch [2][T k]
    int *grp_b = grp_a + 2 * ns;                                  // [2][T k]
    float(*red)[kFusedMaxT] = reinterpret_cast<float(*)[kFusedMaxT]>(grp_b + 2 * ns);
    float *s_amax = reinterpret_cast<float *>(red + kFuRMax * kFuVirt);   // (router sums: [R][8][16]; x maxima: [4][16])
    const int cap = p.slot_cap;
    FuTable tb;
    tb.e = reinterpret_cast<int *>(s_amax + kFusedMaxT);
    tb.cnt = tb.e + (cap + 2);
    tb.off = tb.cnt + (cap + 2);
    tb.bgu = tb.off + (cap + 2);
    tb.bdn = tb.bgu + (cap + 2);
    tb.hdr = tb.bdn + (cap + 2);
    volatile int *abort_flag = tb.hdr + 2;
    volatile int *cfail = tb.hdr + 3;
    volatile int *q_item = tb.hdr + 4;
    uint64_t *bars = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(tb.hdr + kFuHdr) + 7) & ~uintptr_t(7));
    uint64_t *full = bars, *empty = bars + kFuSlotsMax, *table_ready = bars + 2 * kFuSlotsMax;
    uint64_t *q_full = table_ready + 1, *q_empty = q_full + kItemQ;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    const int NX = Cf::kLimbs ? (p.H + kLimbBlockK - 1) / kLimbBlockK : 0;         // x-limb tasks
    const int RE = min(kFuRMax, (p.E + 63) / 64);                                // experts per router task
    const int NR = (p.E + RE - 1) / RE;                                           // router tasks
    const int NH = NX + NR;
    const int A1 = NH + (p.n_shared ? (p.I_sh / kFuRows) * fu_chunks(p.T) : 0);   // first routed gate/up item

    pdl_trigger();   // the next layer's grid may be scheduled: it starts as CTAs of this one exit
    for (int i = tid; i < Cf::kBRow / 4; i += kFfnThreads) reinterpret_cast<uint32_t *>(zrow_sm)[i] = 0u;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init(table_ready, 1);
        for (int q = 0; q < kItemQ; ++q) {
            mbar_init(&q_full[q], 1);
            mbar_init(&q_empty[q], kConsumerWarps);
        }
        tb.hdr[2] = 0;
        tb.hdr[3] = 0;
        for (int w = kFuSeen; w < kFuHdr; ++w) tb.hdr[w] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ======================================================== producer warp
        const uint64_t pol = l2_evict_first_policy();
        FuRing rg = {0, 0u};
        bool ok = true, have_table = false, waited = false;
        unsigned epoch = 0;
        int total = A1;   // a lower bound until the routing is known
        uint32_t unconfirmed = 0, issued_phase = 0;   // bit s: slot s in flight / its parity
        // The claim of the next item is issued one item ahead, so that the atomic's round
        // trip overlaps the current item's stages (lane 0 holds it until the next iteration).
        unsigned claim = 0;
        bool claimed = false;
        auto wait_grid = [&]() {   // the previous grid's writes (x, the workspace) are visible
            if (!waited) {
                pdl_wait();
                epoch = *reinterpret_cast<volatile unsigned *>(ctl_word(p, kCtlEpoch)) + 1u;
                waited = true;
            }
        };
        auto claim_next = [&]() {
            if (!claimed) {
                if (lane == 0) claim = atomicAdd(ctl_word(p, kCtlWork), 1u);
                claimed = true;
            }
        };
        for (int n_item = 0;; ++n_item) {
            int i = blockIdx.x;
            if (n_item > 0) {
                wait_grid();
                claim_next();
                i = G + (int)__shfl_sync(0xffffffffu, claim, 0);
                claimed = false;
            }
            if (ok && i >= A1 && !have_table) {
                wait_grid();
                bool got = true;
                if (lane == 0) got = wait_flag(ctl_word(p, kCtlRoute), epoch, p.status);
                got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                __syncwarp();   // the other lanes read the slot list after lane 0's acquire
                if (got) {
                    fu_build_table(p, tb, cap, A1);
                    total = tb.hdr[1];
                } else {
                    ok = false;
                    if (lane == 0) *abort_flag = 1;
                }
                if (lane == 0) mbar_arrive(table_ready);
                have_table = true;
            }
            const bool done = !ok || i >= total;
            if (lane == 0) {
                const int q = n_item % kItemQ;
                if (!mbar_wait(&q_empty[q], (uint32_t)(((n_item / kItemQ) & 1) ^ 1), p.status)) ok = false;
                q_item[q] = done ? -1 : i;
                mbar_arrive(&q_full[q]);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (done || !ok) break;
            const FuItem it = fu_decode(p, tb, i, NX, NH, A1);
            if (it.kind == 0 || it.kind == 3) continue;   // router / x-limb task: nothing to stream
            // a down item is short: the next claim goes out at once; a gate/up item's claim goes
            // out when its last ring-full of slots does (an item claimed early waits idle
            // behind the current one while other CTAs could have taken it)
            if (waited && it.kind == 2) claim_next();
            const bool gu = it.kind == 1, sh = it.e < 0;
            const int ez = sh ? 0 : it.e;
            const int nkb = (it.K + kLimbBlockK - 1) / kLimbBlockK;
            const int nu = gu ? 2 * nkb : nkb;   // slots of the item
            // what the item's B rows wait for: nothing (routed gate/up: its rows were complete
            // before the routing was published; NVFP4 gate/up once the previous grid is done),
            // the x-limb flag, or the token chunk's flag (unless this CTA saw it already)
            const unsigned *dep = gu ? ((Cf::kLimbs && sh) ? ctl_word(p, kCtlXl) : nullptr) : chunk_flag(p, it.chunk);
            if (!gu && ((tb.hdr[kFuSeen + (it.chunk >> 5)] >> (it.chunk & 31)) & 1)) dep = nullptr;
            // (lane 0 keeps the seen bits: its view decides for the warp)
            const int defer = __shfl_sync(0xffffffffu, (dep || !waited) ? min(nu, S) : 0, 0);
            const CUtensorMap *mA = gu ? (sh ? &maps.sh_g4 : &maps.g4) : (sh ? &maps.sh_d4 : &maps.d4);
            const CUtensorMap *mB = sh ? &maps.sh_u4 : &maps.u4;
            const CUtensorMap *sA = gu ? (sh ? &maps.sh_gb4 : &maps.gb4) : (sh ? &maps.sh_db4 : &maps.db4);
            const CUtensorMap *sB = sh ? &maps.sh_ub4 : &maps.ub4;
            // B row addresses (every lane): a routed item's come from perm (published with the
            // routing); the shared expert's are fixed, so they are known before the grid wait too
            const unsigned char *brow[kFuTok];
            uint32_t bbytes = 0;
#pragma unroll
            for (int j = 0; j < kFuTok; ++j) {
                brow[j] = j < it.ntok ? fu_brow<FMT>(p, it, j) : nullptr;
                bbytes += brow[j] ? (uint32_t)Cf::kBLen : 0u;
            }
            // slot u of the item: gate/up g (u even, with the B rows) or u (odd) of K block
            // u / 2; down: d of K block u (with the B rows)
            auto carries_b = [&](int u) { return !gu || (u & 1) == 0; };
            auto copy_b = [&](int u, int slot) {
                if (!carries_b(u)) return;
                const int kb = gu ? u >> 1 : u;
                unsigned char *dst0 = ring + (size_t)slot * SB + Cf::kBOff;
#pragma unroll
                for (int j = 0; j < kFuTok; ++j)
                    if (brow[j]) bulk_copy(dst0 + j * Cf::kBRow, brow[j] + (size_t)kb * Cf::kBLen, Cf::kBLen, &full[slot]);
            };
            // one slot at ring position (slot, ph): its weight box (and NVFP4 scale box) and, with
            // with_b, its B rows (deferred B rows count in tx too: they land later on the same
            // barrier)
            auto fill = [&](int u, int slot, uint32_t ph, bool with_b) -> bool {
                if (!mbar_wait(&empty[slot], ph ^ 1u, p.status)) return false;
                const uint32_t tx = (uint32_t)(kMatStage + Cf::kScales) + (carries_b(u) ? bbytes : 0u);
                mbar_arrive_expect_tx(&full[slot], tx);
                unsigned char *st = ring + (size_t)slot * SB;
                const int kb = gu ? u >> 1 : u;
                const bool second = gu && (u & 1);
                tma_load_3d(st, second ? mB : mA, &full[slot], kb * kBoxBytes, it.row0, ez, pol);
                if (Cf::kNv)
                    tma_load_3d(st + kMatStage, second ? sB : sA, &full[slot], kb * kBoxBytes / 8, it.row0, ez, pol);
                if (with_b) copy_b(u, slot);
                return true;
            };
            auto issue_unit = [&](int u, bool with_b) -> bool {   // (lane 0)
                if (!fill(u, rg.slot, rg.phase, with_b)) return false;
                issued_phase = (issued_phase & ~(1u << rg.slot)) | (rg.phase << rg.slot);
                unconfirmed |= 1u << rg.slot;
                rg.next(S);
                return true;
            };
            // Slots go out as the ring frees them.  While the B rows' dependency is open a slot
            // carries its weights only (lane 0); the flag is polled once after each such slot
            // (waited for once the item fills the ring), and when it is seen the B rows of the
            // slots so far follow.  The first item may start before the previous grid is done:
            // its weights go out, then the grid wait.  The rest of the item goes out kFuIssue
            // slots at a time, one slot per lane (a single thread's chain of barrier and copy
            // instructions would cap the rate at a few tens of GB/s per CTA).
            const int st0 = rg.slot;
            int u_next = 0;
            if (!waited) {
                if (lane == 0)
                    for (; u_next < defer && ok; ++u_next)
                        if (!issue_unit(u_next, false)) ok = false;
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                wait_grid();
            }
            if (!gu) claim_next();
            const int u_claim = max(0, nu - S);
            int u_par = u_next;   // first slot of the lane-parallel part
            if (lane == 0 && ok) {
                bool have_b = dep == nullptr;
                int b_done = 0;   // slots whose B rows are out (in order)
                auto copy_upto = [&](int n) {   // B rows of slots b_done .. n - 1
                    int slot = st0 + b_done;
                    if (slot >= S) slot -= S;
                    for (; b_done < n; ++b_done) {
                        copy_b(b_done, slot);
                        if (++slot == S) slot = 0;
                    }
                };
                auto seen_now = [&]() {
                    have_b = true;
                    if (!gu) tb.hdr[kFuSeen + (it.chunk >> 5)] |= 1 << (it.chunk & 31);
                };
                if (have_b) copy_upto(u_next);   // (only the grid wait was pending)
                int u = u_next;
                while (!have_b) {
                    // the ring holds as many weight-only slots as it can (or the item's all):
                    // wait for the dependency before anything else goes out
                    if (u >= defer || u >= nu) {
                        if (!wait_flag(dep, epoch, p.status)) { ok = false; break; }
                        seen_now();
                        copy_upto(u);
                        break;
                    }
                    if (gu && u == u_claim) claim_next();
                    if (!issue_unit(u, false)) { ok = false; break; }
                    ++u;
                    if (ld_relaxed(dep) == epoch) {   // one poll per weight-only slot
                        acquire_seen();
                        seen_now();
                        copy_upto(u);
                    }
                }
                u_par = u;
            }
            // lane 0's ring position and bookkeeping to the whole warp
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            u_par = __shfl_sync(0xffffffffu, u_par, 0);
            rg.slot = __shfl_sync(0xffffffffu, rg.slot, 0);
            rg.phase = __shfl_sync(0xffffffffu, rg.phase, 0);
            unconfirmed = __shfl_sync(0xffffffffu, unconfirmed, 0);
            issued_phase = __shfl_sync(0xffffffffu, issued_phase, 0);
            claimed = __shfl_sync(0xffffffffu, claimed ? 1 : 0, 0) != 0;
            for (int u0 = u_par; u0 < nu && ok; u0 += kFuIssue) {
                const int n = min(kFuIssue, nu - u0);
                if (gu && u_claim >= u0 && u_claim < u0 + n) claim_next();
                int slot = rg.slot + lane;
                uint32_t ph = rg.phase;
                if (slot >= S) {
                    slot -= S;
                    ph ^= 1u;
                }
                bool lok = true;
                if (lane < n) lok = fill(u0 + lane, slot, ph, true);
                ok = __all_sync(0xffffffffu, lok);
                const unsigned mine = (lane < n && lok) ? 1u << slot : 0u;
                const unsigned mph = (lane < n && lok) ? ph << slot : 0u;
                const unsigned mask = __reduce_or_sync(0xffffffffu, mine);
                issued_phase = (issued_phase & ~mask) | __reduce_or_sync(0xffffffffu, mph);
                unconfirmed |= mask;
                rg.slot += n;
                if (rg.slot >= S) {
                    rg.slot -= S;
                    rg.phase ^= 1u;
                }
            }
            if (lane == 0 && !ok) *abort_flag = 1;
            // lane 0 decides for the warp (the flag may change between the lanes' reads)
            ok = __shfl_sync(0xffffffffu, (ok && !*abort_flag) ? 1 : 0, 0) != 0;
        }
        if (!have_table && lane == 0) mbar_arrive(table_ready);   // release the consumers (never waited for)
        if (lane == 0 && !ok) {
            // let copies still in flight land before the CTA may exit
            for (int s = 0; s < S; ++s)
                if (unconfirmed >> s & 1u) mbar_wait(&full[s], issued_phase >> s & 1u, p.status, 10000000ull);
        }
        return;
    }

    // ============================================================ consumer warps
    Lane L;
    L.lane = lane;
    L.g = lane >> 2;
    L.tq = lane & 3;
    L.warp = warp;
    L.rw = warp;
    L.ks = 0;
    L.bx = warp;
    L.dk = p.dk;
    {
        const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int lch = lane >> 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) L.off[q] = lrow * kBoxBytes + ((((2 * q + lch) ^ (lrow & 7)) & 7) << 4);
    }
    FuRing rg = {0, 0u};
    bool have_table = false, waited = false;
    unsigned epoch = 0;
    FuPend pend[2];
    pend[0].kind = 0;
    pend[1].kind = 0;
    const uint32_t zsm = smem_u32(zrow_sm);
    __shared__ int s_last;
    for (int n_item = 0;; ++n_item) {
        const int q = n_item % kItemQ;
        int i = -1;
        if (mbar_wait(&q_full[q], (uint32_t)((n_item / kItemQ) & 1), p.status)) {
            i = q_item[q];
        } else {
            *cfail = 1;
            *abort_flag = 1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_empty[q]);
        consumer_sync();
        if (*cfail || i < 0) break;
        if (!waited) {
            if (i >= NX && i < NH) {
                // the router rows are weights: pull them into L2 while the previous grid drains
                const int e0 = (i - NX) * RE, ne = min(RE, p.E - e0);
                const char *row = reinterpret_cast<const char *>(p.wt.router_w + (size_t)e0 * p.H);
                for (int o = tid * 128; o < ne * p.H * 4; o += kFuCT * 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + o));
            }
            pdl_wait();
            epoch = *reinterpret_cast<volatile unsigned *>(ctl_word(p, kCtlEpoch)) + 1u;
            waited = true;
        }
        if (i < NX) {
            // x limb block i; the task completing the set publishes the x-limb flag
            fu_xlimb_task(p, i, tid, red, s_amax);
            if (tid == 0 && atom_inc_acq_rel(ctl_word(p, kCtlXlDone), (unsigned)NX - 1u) == (unsigned)NX - 1u)
                st_release(ctl_word(p, kCtlXl), epoch);
            continue;
        }
        if (i < NH) {
            fu_router_task(p, i - NX, RE, tid, red);
            if (tid == 0) s_last = atom_inc_acq_rel(ctl_word(p, kCtlRouter), (unsigned)NR - 1u) == (unsigned)NR - 1u;
            consumer_sync();
            const bool last = s_last;
            consumer_sync();
            if (last) fu_route_finish<FMT>(p, tid, epoch, s_idx, grp_a, grp_b);
            continue;
        }
        if (i >= A1 && !have_table) {
            if (!mbar_wait(table_ready, 0, p.status)) {
                *cfail = 1;
                *abort_flag = 1;
            }
            consumer_sync();
            if (*cfail) break;
            have_table = true;
        }
        const FuItem it = fu_decode(p, tb, i, NX, NH, A1);
        // a chunk conversion this CTA owes may be what this down item waits for
        if (it.kind == 2 && (pend[0].kind == 1 || pend[1].kind == 1)) fu_advance<FMT>(p, pend, tid, epoch, true);
        bool ok;
        if constexpr (Cf::kLimbs) {
            if (it.kind == 1)
                ok = it.ntok <= 2 ? fu_consume_limbs<true, 1>(p, it, ring, full, empty, rg, L, zsm, pend, cfail,
                                                              abort_flag, tb, epoch)
                                  : fu_consume_limbs<true, 3>(p, it, ring, full, empty, rg, L, zsm, pend, cfail,
                                                              abort_flag, tb, epoch);
            else
                ok = it.ntok <= 2 ? fu_consume_limbs<false, 1>(p, it, ring, full, empty, rg, L, zsm, pend, cfail,
                                                               abort_flag, tb, epoch)
                                  : fu_consume_limbs<false, 3>(p, it, ring, full, empty, rg, L, zsm, pend, cfail,
                                                               abort_flag, tb, epoch);
        } else {
            ok = it.kind == 1 ? fu_consume_nv<true>(p, it, ring, full, empty, rg, L, zsm, pend, cfail, abort_flag, tb,
                                                    epoch)
                              : fu_consume_nv<false>(p, it, ring, full, empty, rg, L, zsm, pend, cfail, abort_flag, tb,
                                                     epoch);
        }
        if (!ok) break;
    }
    if (!*cfail) fu_advance<FMT>(p, pend, tid, epoch, true);
    if (!waited) {   // a CTA without items still reads the epoch before counting itself done
        pdl_wait();
        epoch = *reinterpret_cast<volatile unsigned *>(ctl_word(p, kCtlEpoch)) + 1u;
    }
    // the last CTA to finish resets the claim counters and closes the call's epoch (every
    // producer has made its last claim before its consumers saw the end of the queue)
    if (tid == 0 && !*cfail && atomicAdd(ctl_word(p, kCtlDone), 1u) == (unsigned)G - 1u) {
        atomicExch(ctl_word(p, kCtlWork), 0u);
        atomicExch(ctl_word(p, kCtlDone), 0u);
        atomicExch(ctl_word(p, kCtlEpoch), epoch);
    }
}

// ------------------------------------------------------------------ host side
constexpr size_t kFuSmemPerCta = 112 * 1024;   // two CTAs per SM

// Ring geometry of a launch: slots of one weight box (+ scale box) and one K block of the
// B rows of min(T, 8) tokens, as many as fit beside the fixed part (at most kFuSlotsMax).
template <int FMT>
static void fused_geometry(const FusedParams &p, int &slots, int &slot_bytes, int &cap, size_t &smem)
{
    using Cf = FuCfg<FMT>;
    const int nb = p.T < kFuTok ? p.T : kFuTok;
    cap = p.E < p.T * p.k ? p.E : p.T * p.k;
    slot_bytes = (Cf::kBOff + nb * Cf::kBRow + 1023) / 1024 * 1024;
    const size_t fixed = fu_fixed_smem<FMT>(cap, p.T * p.k);
    int n = fixed < kFuSmemPerCta ? (int)((kFuSmemPerCta - fixed) / slot_bytes) : 0;
    slots = n < 4 ? 4 : (n > kFuSlotsMax ? kFuSlotsMax : n);
    smem = fixed + (size_t)slots * slot_bytes;
}

template <int FMT>
static cudaError_t fused_prepare_t(int *blocks_per_sm)
{
    int dev = 0, optin = 0;
    cudaFuncAttributes fa;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, fused_kernel<FMT>);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fused_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fused_kernel<FMT>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, fused_kernel<FMT>, kFfnThreads, kFuSmemPerCta);
}

// Resident CTAs per SM of the fused kernel of a format (the grid must not exceed what is
// resident at once: its CTAs wait for one another's flags).
cudaError_t fused_prepare(int fmt, int *blocks_per_sm)
{
    return fmt == MOE_FMT_NVFP4 ? fused_prepare_t<MOE_FMT_NVFP4>(blocks_per_sm)
                                : fused_prepare_t<MOE_FMT_INT4_ROWSCALE>(blocks_per_sm);
}

template <int FMT>
static cudaError_t launch_fused_t(const LayerMaps &maps, const FusedParams &p0, int grid, bool pdl, cudaStream_t s)
{
    FusedParams p = p0;
    size_t smem = 0;
    fused_geometry<FMT>(p, p.stages, p.stage_bytes, p.slot_cap, smem);
    if (smem > kFuSmemPerCta) return cudaErrorInvalidValue;   // (T k too large for the layout)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kFfnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, fused_kernel<FMT>, maps, p);
}

cudaError_t launch_fused(const LayerMaps &maps, const FusedParams &p, int grid, bool pdl, cudaStream_t s)
{
    return p.fmt == MOE_FMT_NVFP4 ? launch_fused_t<MOE_FMT_NVFP4>(maps, p, grid, pdl, s)
                                  : launch_fused_t<MOE_FMT_INT4_ROWSCALE>(maps, p, grid, pdl, s);
}

}  // namespace moe
