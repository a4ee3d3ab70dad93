// moe_ffn.cu -- expert FFN for decode-sized batches: gate/up and down projections on
// 4-bit weights (int4 with per-row scales, or NVFP4), dequantised in registers inside
// the matmul, fp16 activations, fp32 accumulation.
//
// Sources: W4A16 (INT4 weights, FP16 activations) and small-batch custom kernels:
// "GLM-5.3-Flash 320B MoEを4枚のCMP 170HXで動かすvLLMレシピ" (648news); int4 with per-row
// scales and the batch MoE union (each unique expert read once for all its tokens):
// "Show HN: 低速のコンピュータでGLM 5.2を動かす方法" (hakusoku), 実装済み機能; NVFP4
// decoded in registers, never expanded to fp16 in memory: "GTX 1070向け35Bパラメータ
// MoEモデル推論エンジン公開" (648news), "VRAMとシステムメモリで重みを分割する設計".
//
// Design (B200).  The weight stream is the whole cost (2 flop per weight per token), so
// every byte is read from HBM once, by TMA, into a ring of shared-memory stages, while
// four consumer warps turn nibbles into fp16 in registers and feed mma.sync m16n8k16:
// the tensor cores serve as a wide dot-product engine (256 weights per instruction),
// which keeps the issue slots below the HBM rate -- CUDA-core FMA would need about three
// instructions per weight and fall behind.
//
// Warp layout RW x KS (RW * KS = 4 consumer warps).  A work item is (expert slot, 16*RW
// output rows, up to 32 tokens).  Warp (rw, ks) owns rows [16 rw, 16 rw + 16) of the
// item and K-box ks of every stage.  A stage holds, per matrix, RW*KS boxes of
// 16 rows x 128 bytes (128-byte swizzle), i.e. 8 KB.  With KS = 1 every warp covers the
// whole K of its rows, so the epilogue runs from registers with no cross-warp traffic;
// with KS = 4 (small layers, to make enough items) the four K-slices are reduced in a
// fixed order through shared memory.  The host picks RW per launch for load balance.
// A persistent grid walks the items with a fixed stride, so results never depend on
// timing.
//
// gate/up: h = SiLU(g * sg) * (u * su) rounded to fp16, stored per bucket position with
//          every 8-column group in the down kernel's B-fragment order.
// down:    y_assign[a] = (W_d h) * sd in fp32 (and the shared expert's y_shared); a
//          separate combine kernel forms y = shared + sum_j w_j y_assign.
//
// Programmatic dependent launch: the gate/up kernel runs the shared expert (no routing
// needed) before griddepcontrol.wait; the down kernel's producer streams weights before
// its consumers wait for h.
#include <cuda_fp16.h>
#include <math.h>

#include "moe_device.cuh"
#include "moe_expert.cuh"
#include "moe_internal.h"

namespace moe {


struct SlotTable {
    int *e;      // expert id, -1 = shared expert
    int *cnt;    // tokens in the bucket
    int *off;    // bucket start (position in perm)
    int *base;   // first item of the slot; base[n_slots] = total
    int *hdr;    // [0] n_slots, [1] total items, [2] producer abort, [3] consumer fail
};

struct Item {
    int e;        // expert, -1 = shared
    int row0;     // first output row of the item
    int tok0;     // first bucket position of the chunk (relative to the bucket)
    int ntok;     // tokens in the chunk (1..32)
    int boff;     // bucket start in perm order
    int K;        // input dimension of the matrix
};

template <bool GU>
__device__ __forceinline__ int slot_rows(const FfnParams &p, bool shared)
{
    return GU ? (shared ? p.I_sh : p.I) : p.H;
}
template <bool GU>
__device__ __forceinline__ int slot_K(const FfnParams &p, bool shared)
{
    return GU ? p.H : (shared ? p.I_sh : p.I);
}

template <bool GU, int RW>
__device__ __forceinline__ int shared_items(const FfnParams &p)
{
    if (!p.n_shared) return 0;
    return (slot_rows<GU>(p, true) / (kRowTile * RW)) * ((p.T + p.tok_chunk - 1) / p.tok_chunk);
}

template <bool GU, int RW>
__device__ __forceinline__ Item make_item(const FfnParams &p, int e, int cnt, int boff, int local)
{
    const bool shared = e < 0;
    const int tiles = slot_rows<GU>(p, shared) / (kRowTile * RW);
    Item it;
    it.e = e;
    it.row0 = (local % tiles) * kRowTile * RW;
    it.tok0 = (local / tiles) * p.tok_chunk;
    it.ntok = min(p.tok_chunk, cnt - it.tok0);
    it.boff = boff;
    it.K = slot_K<GU>(p, shared);
    return it;
}

template <bool GU, int RW>
__device__ Item decode_item(const FfnParams &p, const SlotTable &tb, int i)
{
    int lo = 0, hi = tb.hdr[0] - 1;   // last slot whose first item is <= i
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb.base[mid] <= i) lo = mid;
        else hi = mid - 1;
    }
    return make_item<GU, RW>(p, tb.e[lo], tb.cnt[lo], tb.off[lo], i - tb.base[lo]);
}

// Slot table: the shared expert first, then the non-empty experts in ascending order,
// from the router's compact list when present, else by scanning the offsets.  One warp.
template <bool GU, int RW>
__device__ void build_slot_table(const FfnParams &p, const SlotTable &tb, int E)
{
    const int lane = threadIdx.x & 31;
    int ns = 0, acc = 0;
    if (p.n_shared) {
        if (lane == 0) {
            tb.e[0] = -1;
            tb.cnt[0] = p.T;
            tb.off[0] = 0;
            tb.base[0] = 0;
        }
        ns = 1;
        acc = shared_items<GU, RW>(p);
    }
    const int tiles = slot_rows<GU>(p, false) / (kRowTile * RW);
    // with the router's slot list, its first 32 entries are read together with its length
    int4 s0 = make_int4(-1, 0, 0, 0);
    if (p.slots && lane < E) s0 = __ldcg(p.slots + lane);
    const int n_scan = p.unique ? min(__ldcg(p.n_unique), E) : E;
    for (int b = 0; b < n_scan; b += 32) {
        const int j = b + lane;
        int e = -1, cnt = 0, off = 0;
        if (j < n_scan) {
            if (p.slots) {
                const int4 sj = b == 0 ? s0 : __ldcg(p.slots + j);
                e = sj.x;
                cnt = sj.y;
                off = sj.z;
            } else {
                e = p.unique ? __ldcg(p.unique + j) : j;
                if (e >= 0 && e < E) {
                    off = __ldcg(p.offsets + e);
                    cnt = __ldcg(p.offsets + e + 1) - off;
                }
            }
            if (e < 0 || e >= E || off < 0 || cnt < 0 || off + cnt > p.T * p.k) {
                if (p.unique || cnt != 0) record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                cnt = 0;
            }
        }
        const bool has = cnt > 0;
        const unsigned bal = __ballot_sync(0xffffffffu, has);
        const int nit = has ? tiles * ((cnt + p.tok_chunk - 1) / p.tok_chunk) : 0;
        int incl = nit;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (has) {
            const int pos = ns + __popc(bal & ((1u << lane) - 1u));
            tb.e[pos] = e;
            tb.cnt[pos] = cnt;
            tb.off[pos] = off;
            tb.base[pos] = acc + incl - nit;
        }
        ns += __popc(bal);
        acc += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        tb.base[ns] = acc;
        tb.hdr[0] = ns;
        tb.hdr[1] = acc;
    }
    __syncwarp();
}

// B-operand row of bucket column `col` of an item: an x row (gate/up; the permuted copy
// unless perm_b) or an h row (down); NULL for padding columns or a bad index
template <bool GU>
__device__ __forceinline__ const uint16_t *item_brow(const FfnParams &p, const Item &it, int col, bool perm_b)
{
    if (col >= it.ntok) return nullptr;
    const bool sh = it.e < 0;
    const int bpos = it.tok0 + col;
    if (GU) {
        int t = bpos;
        if (!sh) {
            const int a = __ldg(p.perm + it.boff + bpos);
            t = (a >= 0 && a < p.T * p.k) ? a / p.k : -1;
            if (t < 0) {
                record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                return nullptr;
            }
        }
        return (perm_b ? p.x : p.xb) + (size_t)t * p.H;
    }
    return sh ? reinterpret_cast<const uint16_t *>(p.h_sh) + (size_t)bpos * p.I_sh
              : reinterpret_cast<const uint16_t *>(p.h) + (size_t)(it.boff + bpos) * p.I;
}

// bytes of one limb row of a K-long operand
__device__ __forceinline__ size_t limb_row_bytes(int K)
{
    return (size_t)((K + kLimbBlockK - 1) / kLimbBlockK) * kLimbBlockBytes;
}

// int8 path: limb row of bucket column `col` of an item (x limbs for gate/up, h limbs for
// down); NULL for padding columns or a bad index
template <bool GU>
__device__ __forceinline__ const unsigned char *item_brow_limbs(const FfnParams &p, const Item &it, int col)
{
    if (col >= it.ntok) return nullptr;
    const bool sh = it.e < 0;
    const int bpos = it.tok0 + col;
    if (GU) {
        int t = bpos;
        if (!sh) {
            const int a = __ldg(p.perm + it.boff + bpos);
            t = (a >= 0 && a < p.T * p.k) ? a / p.k : -1;
            if (t < 0) {
                record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                return nullptr;
            }
        }
        return p.x_limbs + (size_t)t * limb_row_bytes(p.H);
    }
    return sh ? p.hsh_limbs + (size_t)bpos * limb_row_bytes(p.I_sh)
              : p.h_limbs + (size_t)(it.boff + bpos) * limb_row_bytes(p.I);
}

// One warp's share of one work item: the stages of the item (for each stage the B
// fragments of the warp's K range are fetched before its weights are waited for, since
// they do not depend on them), then the epilogue.  NN: n-tiles of 8 tokens.  PERM: the
// int4 gate/up B operand arrives in natural order and is permuted here to the dequant
// pair order (0,4)(1,5)(2,6)(3,7); otherwise it is already in fragment order.
// Returns false (every consumer warp alike) when a wait gave up.
template <int FMT, bool GU, int KS, int NNMAX, int NN, bool PERM>
__device__ __forceinline__ bool consume_item(const FfnParams &p, const SlotTable tb, const Item it,
                                          unsigned char *ring, unsigned char *bring, uint64_t *full, uint64_t *empty,
                                          int &stage, uint32_t &phase, const Lane L, const BRows brow, uint32_t zsm,
                                          float *red, volatile int *cfail, volatile int *abort_flag)
{
    using C = FfnCfg<FMT, GU, KS, NNMAX>;
    const int S = p.stages;
    constexpr int RW = C::kRW;
    const bool sh = it.e < 0;
    const int Kb = it.K / 2;
    const int nst = (Kb + C::kStageK - 1) / C::kStageK;
    constexpr int P = Chains<NN>::P;
    float part[C::kMats][NN][P][4];
#pragma unroll
    for (int m = 0; m < C::kMats; ++m)
#pragma unroll
        for (int n = 0; n < NN; ++n)
#pragma unroll
            for (int j = 0; j < P; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) part[m][n][j][c] = 0.f;

    bool ok = true;
    if constexpr (C::kSmemB) {
        // B fragments from the stage's token rows in shared memory (padding lanes read
        // the zero row)
        for (int s = 0; s < nst; ++s) {
            const int kbox = s * C::kStageK;
            if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
            const unsigned char *st = ring + (size_t)stage * C::kStageBytes;
            const uint32_t abase = smem_u32(st + L.bx * kBoxSmem);
            const uint32_t bsm =
                (L.g < it.ntok ? smem_u32(bring + (size_t)stage * p.b_stage + L.g * C::kBRow) : zsm) + 16 * L.tq;
            if (kbox + kBoxBytes <= Kb) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    chunk_pair<FMT, GU, KS, NN, PERM>(st, abase, L, q, 0, lds128(bsm + 128 * q),
                                                      lds128(bsm + 128 * q + 64), brow, part);
            } else {
                const int npairs = kbox < Kb ? (Kb - kbox) / 32 : 0;
                for (int q = 0; q < npairs; ++q)
                    chunk_pair<FMT, GU, KS, NN, PERM>(st, abase, L, q, 0, lds128(bsm + 128 * q),
                                                      lds128(bsm + 128 * q + 64), brow, part);
            }
            __syncwarp();
            if (L.lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == S) { stage = 0; phase ^= 1u; }
        }
    } else
    for (int s = 0; s < nst; ++s) {
        const int kbox = s * C::kStageK + L.ks * kBoxBytes;     // K byte of this warp's box
        const uint16_t *b0 = brow.r[0] + 2 * kbox + 8 * L.tq;
        if (kbox + kBoxBytes <= Kb) {
            // full box: four chunk pairs, fully unrolled
            uint4 xb[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) xb[c] = __ldg(reinterpret_cast<const uint4 *>(b0 + 32 * c));
            if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
            const unsigned char *st = ring + (size_t)stage * C::kStageBytes;
            const uint32_t abase = smem_u32(st + L.bx * kBoxSmem);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                chunk_pair<FMT, GU, KS, NN, PERM>(st, abase, L, q, 2 * kbox + 64 * q, xb[2 * q], xb[2 * q + 1], brow, part);
        } else {
            // the last, partial box (or none): K is a multiple of 64, so whole chunk pairs
            if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
            const unsigned char *st = ring + (size_t)stage * C::kStageBytes;
            const uint32_t abase = smem_u32(st + L.bx * kBoxSmem);
            const int npairs = kbox < Kb ? (Kb - kbox) / 32 : 0;
            for (int q = 0; q < npairs; ++q) {
                const uint4 x0 = __ldg(reinterpret_cast<const uint4 *>(b0 + 64 * q));
                const uint4 x1 = __ldg(reinterpret_cast<const uint4 *>(b0 + 64 * q + 32));
                chunk_pair<FMT, GU, KS, NN, PERM>(st, abase, L, q, 2 * kbox + 64 * q, x0, x1, brow, part);
            }
        }
        __syncwarp();
        if (L.lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == S) { stage = 0; phase ^= 1u; }
    }
    if (!ok) {
        *cfail = 1;
        *abort_flag = 1;
    }
    // the partial chains, summed in a fixed order
    float acc[C::kMats][NN][4];
#pragma unroll
    for (int m = 0; m < C::kMats; ++m)
#pragma unroll
        for (int n = 0; n < NN; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v = part[m][n][0][c];
#pragma unroll
                for (int j = 1; j < P; ++j) v += part[m][n][j][c];
                acc[m][n][c] = v;
            }

    const int rows_all = slot_rows<GU>(p, sh);
    const float *sc0 = GU ? (sh ? p.wt.sh_g_scale : p.wt.g_scale) : (sh ? p.wt.sh_d_scale : p.wt.d_scale);
    const float *sc1 = sh ? p.wt.sh_u_scale : p.wt.u_scale;
    const int tid = threadIdx.x;
    if constexpr (KS == 1) {
        // ------------------------------------------------ epilogue from registers
        consumer_sync();   // only to agree on failure: all warps ran the same stages
        if (*cfail) return false;
#pragma unroll
        for (int n = 0; n < NN; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int col = 8 * n + 2 * L.tq + (c & 1);
                if (col >= it.ntok) continue;
                const int row = it.row0 + L.rw * kRowTile + L.g + (c >> 1) * 8;
                const int bpos = it.tok0 + col;
                if (GU) {
                    const float gv = acc[0][n][c] * mat_scale<FMT>(sc0, it.e, rows_all, row);
                    const float uv = acc[C::kMats - 1][n][c] * mat_scale<FMT>(sc1, it.e, rows_all, row);
                    const float hv = gv / (1.f + expf(-gv)) * uv;
                    __half *dst = sh ? p.h_sh + (size_t)bpos * p.I_sh : p.h + (size_t)(it.boff + bpos) * p.I;
                    dst[h_pos<FMT>(row)] = __float2half_rn(hv);
                } else {
                    const float yv = acc[0][n][c] * mat_scale<FMT>(sc0, it.e, rows_all, row);
                    if (sh) {
                        p.y_shared[(size_t)bpos * p.H + row] = yv;
                    } else {
                        const int a = __ldg(p.perm + it.boff + bpos);
                        if (a >= 0 && a < p.T * p.k) p.y_assign[(size_t)a * p.H + row] = yv;
                        else record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                    }
                }
            }
    } else {
        // ------------------------------------------------ K-split epilogue (KS = 4)
        // partial sums of the four K-slices -> shared memory [warp][mat][col][row]
#pragma unroll
        for (int m = 0; m < C::kMats; ++m)
#pragma unroll
            for (int n = 0; n < NN; ++n) {
                float *r = red + ((L.warp * C::kMats + m) * kTokChunk) * kRowTile;
                const int c0 = 8 * n + 2 * L.tq;
                r[c0 * kRowTile + L.g] = acc[m][n][0];
                r[(c0 + 1) * kRowTile + L.g] = acc[m][n][1];
                r[c0 * kRowTile + L.g + 8] = acc[m][n][2];
                r[(c0 + 1) * kRowTile + L.g + 8] = acc[m][n][3];
            }
        consumer_sync();
        if (*cfail) return false;
        for (int o = tid; o < it.ntok * kRowTile; o += kConsumerWarps * 32) {
            const int r = o % kRowTile, col = o / kRowTile;
            const int row = it.row0 + r;
            float v0 = 0.f, v1 = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                v0 += red[((w * C::kMats + 0) * kTokChunk + col) * kRowTile + r];
                if (GU) v1 += red[((w * C::kMats + 1) * kTokChunk + col) * kRowTile + r];
            }
            const int bpos = it.tok0 + col;
            if (GU) {
                const float gv = v0 * mat_scale<FMT>(sc0, it.e, rows_all, row);
                const float uv = v1 * mat_scale<FMT>(sc1, it.e, rows_all, row);
                const float hv = gv / (1.f + expf(-gv)) * uv;
                __half *dst = sh ? p.h_sh + (size_t)bpos * p.I_sh : p.h + (size_t)(it.boff + bpos) * p.I;
                dst[h_pos<FMT>(row)] = __float2half_rn(hv);
            } else {
                const float yv = v0 * mat_scale<FMT>(sc0, it.e, rows_all, row);
                if (sh) {
                    p.y_shared[(size_t)bpos * p.H + row] = yv;
                } else {
                    const int a = __ldg(p.perm + it.boff + bpos);
                    if (a >= 0 && a < p.T * p.k) p.y_assign[(size_t)a * p.H + row] = yv;
                    else record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                }
            }
        }
        consumer_sync();
    }
    (void)RW;
    return true;
}

// A completion counter increment whose result is looked at later: gate/up on the int8
// path counts each finished row tile of a token chunk at the end of an item and settles
// it after the next item's stages; the CTA that completes the chunk converts its h rows.
struct Pending {
    int kind;          // 0 none, 1 h chunk
    unsigned old, target;
    int sh, tok0, ntok, boff;
};

template <bool GU, int NT = kConsumerWarps * 32, int BAR = 1>
__device__ __forceinline__ void settle(const FfnParams &p, Pending &pd, int ltid)
{
    if (pd.kind == 1) {
        __shared__ int s_conv;
        if (ltid == 0) s_conv = pd.old == pd.target;
        consumer_sync<NT, BAR>();
        if (s_conv) {
            if (pd.sh)
                convert_h_rows<NT, BAR>(p.h_sh + (size_t)pd.tok0 * p.I_sh, p.I_sh, p.hsh_limbs + (size_t)pd.tok0 * limb_row_bytes(p.I_sh),
                               p.hsh_limb_scale + pd.tok0, p.h_amax + p.T * p.k + pd.tok0, pd.ntok, p.I_sh, ltid);
            else
                convert_h_rows<NT, BAR>(p.h + (size_t)(pd.boff + pd.tok0) * p.I, p.I,
                               p.h_limbs + (size_t)(pd.boff + pd.tok0) * limb_row_bytes(p.I),
                               p.h_limb_scale + pd.boff + pd.tok0, p.h_amax + pd.boff + pd.tok0, pd.ntok, p.I, ltid);
        }
    }
    pd.kind = 0;
}

// One warp's share of one work item on the int8 path (int8, int4 or int2 weights, KS = 1,
// at most 8 tokens): the stages, then the epilogue.  NN = 1 for items of 1-2 tokens, 3
// otherwise.  The accumulators hold 2^shift x sum(code * limb) per (limb, token) (shift
// 0, 4, 6 for int8, int4, int2); the epilogue forms
// sum(code * X) = S0 + 256 S1 + 65536 S2 exactly in 64-bit integers and scales it by
// 2^-sh and the row scale in fp64.  Gate/up then stores h in fp16 and the last item of
// a token chunk converts the chunk's h rows to limbs for the down kernel.  Everything
// the epilogue needs besides the accumulators is loaded before the stages.
template <int FMT, bool GU, int NN>
__device__ __forceinline__ bool consume_item_limbs(const FfnParams &p, const SlotTable tb, const Item it,
                                                   unsigned char *ring, unsigned char *bring, uint64_t *full,
                                                   uint64_t *empty, int &stage, uint32_t &phase, const Lane L,
                                                   uint32_t zsm, Pending &pd, volatile int *cfail,
                                                   volatile int *abort_flag)
{
    using C = FfnCfg<FMT, GU, 1, 1>;
    const int S = p.stages;
    constexpr int M = C::kMats;
    const bool sh = it.e < 0;
    const int nst = (it.K + C::kStageVals - 1) / C::kStageVals;
    // this lane's B column in n-tile 0: (limb, token); its limb block of each stage sits in
    // the stage's B rows (padding columns read the zero row)
    const int lcol = NN == 1 ? (L.g >> 1) : 0;
    const int tcol = NN == 1 ? (L.g & 1) : L.g;
    const bool bval = lcol < 3 && tcol < it.ntok;
    const uint32_t boff = (uint32_t)(tcol * C::kBRow + lcol * kLimbBlockK + 16 * L.tq);

    // epilogue operands: row scales of rows g and g + 8, and for the lane's two output
    // tokens (u = c & 1) the assignment id (routed) and the activation scale
    const int rows_all = slot_rows<GU>(p, sh);
    const int ez = sh ? 0 : it.e;
    const int rowA = it.row0 + L.rw * kRowTile + L.g;
    const float *sc0 = GU ? (sh ? p.wt.sh_g_scale : p.wt.g_scale) : (sh ? p.wt.sh_d_scale : p.wt.d_scale);
    const float *sc1 = sh ? p.wt.sh_u_scale : p.wt.u_scale;
    float rs0[2], rs1[2] = {0.f, 0.f}, xsc[2] = {0.f, 0.f};
    int asg[2];
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
        const int bpos = it.tok0 + t;
        asg[u] = (uval[u] && !sh) ? __ldg(p.perm + it.boff + bpos) : bpos;
        if (!GU && uval[u]) xsc[u] = __ldcg(sh ? p.hsh_limb_scale + bpos : p.h_limb_scale + it.boff + bpos);
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
    for (int s = 0; s < nst; ++s) {
        // 64-value groups of this stage (K is a multiple of 64)
        const int ngroups = min(C::kGroups, (it.K - s * C::kStageVals) / 64);
        if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
        const uint32_t bb = bval ? smem_u32(bring + (size_t)stage * p.b_stage) + boff : zsm + 16 * L.tq;
        // (the zero row is one stage's B row long: every group's offset stays inside it)
        if (GU && s == 0) {
            // the activation scales of the lane's tokens (their ids came with the perm loads)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int a = asg[u];
                const int tok = sh ? a : ((a >= 0 && a < p.T * p.k) ? a / p.k : -1);
                if (uval[u] && tok >= 0) xsc[u] = __ldcg(p.x_limb_scale + tok);
            }
        }
        const uint32_t abase = smem_u32(ring + (size_t)stage * C::kStageBytes + L.bx * kBoxSmem);
        // the groups of one 256-value limb block at a time (int2 stages hold two blocks)
#pragma unroll
        for (int blk = 0; blk < C::kGroups / 4; ++blk) {
            uint4 B[4][NN];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int n = 0; n < NN; ++n) B[q][n] = lds128(bb + blk * kLimbBlockBytes + n * kLimbBlockK + 64 * q);
            if (ngroups == C::kGroups) {
#pragma unroll
                for (int q = 0; q < 4; ++q) chunk_pair_limbs<FMT, GU, NN>(abase, L, 4 * blk + q, B[q], acc2);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (4 * blk + q < ngroups) chunk_pair_limbs<FMT, GU, NN>(abase, L, 4 * blk + q, B[q], acc2);
            }
        }
        __syncwarp();
        if (L.lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == S) { stage = 0; phase ^= 1u; }
    }
    if (!ok) {
        *cfail = 1;
        *abort_flag = 1;
    }
    if (GU) {
        // the previous item's completion check, now that its atomic has long returned
        // (its h conversion is a CTA-wide step), then agreement on failure
        settle<GU>(p, pd, threadIdx.x);
        consumer_sync();
        if (*cfail) return false;
    } else {
        // down: the warps own disjoint rows and meet at no barrier; a warp whose wait gave
        // up leaves, and the others end at their own bounded waits (the producer stops)
        if (!ok) return false;
    }

    int acc[M][NN][4];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int n = 0; n < NN; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[m][n][c] = acc2[0][m][n][c] + acc2[1][m][n][c];
    float hmax[2] = {0.f, 0.f};   // gate/up: largest |h| (as stored) of the lane's tokens
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        long long Sv[M];
        if constexpr (NN == 1) {
            // lanes tq = 0, 1, 2 of a quad hold limbs 0, 1, 2 of tokens c & 1
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const int v0 = acc[m][0][c] >> C::kCodeShift;
                const int v1 = __shfl_down_sync(0xffffffffu, v0, 1);
                const int v2 = __shfl_down_sync(0xffffffffu, v0, 2);
                Sv[m] = (long long)v0 + 256ll * v1 + 65536ll * v2;
            }
        } else {
#pragma unroll
            for (int m = 0; m < M; ++m)
                Sv[m] = (long long)(acc[m][0][c] >> C::kCodeShift) + 256ll * (acc[m][1][c] >> C::kCodeShift) +
                        65536ll * (acc[m][2][c] >> C::kCodeShift);
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
            if constexpr (NN == 1) {
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            } else {
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            }
            const int t = NN == 1 ? u : 2 * L.tq + u;
            if (L.g == 0 && (NN == 1 ? L.tq == 0 : true) && t < it.ntok)
                atomicMax(p.h_amax + (sh ? p.T * p.k : it.boff) + it.tok0 + t, __float_as_uint(m));
        }
        // count this row tile of the token chunk; the last one converts the chunk's h rows
        consumer_sync();
        pd.kind = 1;
        pd.sh = sh;
        pd.tok0 = it.tok0;
        pd.ntok = it.ntok;
        pd.boff = it.boff;
        pd.target = (unsigned)(rows_all / (kRowTile * C::kRW)) - 1u;
        if (threadIdx.x == 0) {
            const int idx = sh ? p.T * p.k + it.tok0 : it.boff + it.tok0;
            pd.old = atom_inc_acq_rel(p.chunk_counters + idx, pd.target);
        }
    }
    return true;
}

template <int FMT, bool GU, int KS, int NNMAX>
__global__ void __launch_bounds__(kFfnThreads, ffn_min_ctas<FMT, GU, KS, NNMAX>()) ffn_kernel(const __grid_constant__ LayerMaps maps,
                                                          const FfnParams p)
{
    using C = FfnCfg<FMT, GU, KS, NNMAX>;
    constexpr int RW = C::kRW;
    const int S = p.stages;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *ring = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *bring = ring + (size_t)S * C::kStageBytes;            // per-stage B rows (decode variant)
    unsigned char *zrow_sm = bring + (size_t)S * p.b_stage;
    float *red = reinterpret_cast<float *>(zrow_sm + C::kZeroRow);
    int *tbl = reinterpret_cast<int *>(red + C::kRedFloats);
    const int E = p.E;
    SlotTable tb;
    tb.e = tbl;
    tb.cnt = tbl + (E + 2);
    tb.off = tbl + 2 * (E + 2);
    tb.base = tbl + 3 * (E + 2);
    tb.hdr = tbl + 4 * (E + 2);
    volatile int *abort_flag = tb.hdr + 2;
    volatile int *cfail = tb.hdr + 3;
    volatile int *q_item = tb.hdr + 4;   // [kItemQ] announced work items (-1: no more)
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(tb.hdr + 16) + 7) & ~uintptr_t(7));
    uint64_t *full = bars, *empty = bars + S, *table_ready = bars + 2 * kStagesMax;
    uint64_t *q_full = table_ready + 1, *q_empty = q_full + kItemQ;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    // the combine kernel after the down kernel may start at once: it waits for this grid
    if constexpr (!GU) pdl_trigger();
    // Only the gate/up kernel runs shared-expert items before the slot table exists (they
    // need no routing).  The down kernel builds its table at once (no wait involved).
    const int n_pre = GU ? shared_items<GU, RW>(p) : 0;
    // Work items are claimed from a global counter by each CTA's producer warp (items
    // differ in cost with their token counts) and announced to the consumer warps through
    // a small queue; the last CTA to finish resets the counters for the next launch.

    for (int i = tid; i < C::kZeroRow / 4; i += kFfnThreads) reinterpret_cast<uint32_t *>(zrow_sm)[i] = 0u;
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
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ======================================================== producer warp
        // whole-K launches (KS = 1) fetch the four warps' 64 rows of a matrix in one box
        constexpr bool kBox64 = KS == 1;
        const CUtensorMap *mA0 = kBox64 ? (GU ? &maps.g4 : &maps.d4) : (GU ? &maps.g : &maps.d);
        const CUtensorMap *mA1 = kBox64 ? &maps.u4 : &maps.u;
        const CUtensorMap *mS0 = kBox64 ? (GU ? &maps.sh_g4 : &maps.sh_d4) : (GU ? &maps.sh_g : &maps.sh_d);
        const CUtensorMap *mS1 = kBox64 ? &maps.sh_u4 : &maps.sh_u;
        const CUtensorMap *bA0 = kBox64 ? (GU ? &maps.gb4 : &maps.db4) : (GU ? &maps.gb : &maps.db);
        const CUtensorMap *bA1 = kBox64 ? &maps.ub4 : &maps.ub;
        const CUtensorMap *bS0 = kBox64 ? (GU ? &maps.sh_gb4 : &maps.sh_db4) : (GU ? &maps.sh_gb : &maps.sh_db);
        const CUtensorMap *bS1 = kBox64 ? &maps.sh_ub4 : &maps.sh_ub;
        const uint64_t pol = l2_evict_first_policy();
        int stage = 0;
        uint32_t phase = 0;
        // gate/up needs nothing from the router for its shared-expert items, except on the
        // int8 path, whose x limbs the router writes: their B copies wait like h's do
        bool ok = true, have_table = false, pdl_done = GU && !C::kLimbs;
        int total = n_pre;
        uint32_t unconfirmed = 0, issued_phase = 0;   // bit s: stage s in flight / its parity
        for (int n_item = 0;; ++n_item) {
            // claimed only when this CTA can start it (its ring still holds the previous
            // item's last stages, which cover the atomic's round trip)
            const int i = (int)__shfl_sync(0xffffffffu, lane == 0 ? atomicAdd(p.work, 1u) : 0u, 0);
            if (ok && i >= n_pre && !have_table) {
                if (GU) {
                    pdl_wait();
                    pdl_done = true;
                }
                build_slot_table<GU, RW>(p, tb, E);
                if (lane == 0) mbar_arrive(table_ready);
                have_table = true;
                total = tb.hdr[1];
                if (GU) pdl_trigger();
            }
            const bool done = !ok || i >= total;
            if (lane == 0) {
                // announce item i (or the end) to the consumers
                const int q = n_item % kItemQ;
                if (!mbar_wait(&q_empty[q], (uint32_t)(((n_item / kItemQ) & 1) ^ 1), p.status)) ok = false;
                q_item[q] = done ? -1 : i;
                mbar_arrive(&q_full[q]);
            }
            if (done) break;
            if (lane == 0 && ok) {
                const Item it = (i < n_pre) ? make_item<GU, RW>(p, -1, p.T, 0, i) : decode_item<GU, RW>(p, tb, i);
                const bool sh = it.e < 0;
                const int ez = sh ? 0 : it.e;
                const int Kb = it.K * code_bits(FMT) / 8;   // code bytes of a row
                if constexpr (C::kLimbs) {
                    // the item's row scales, needed by its epilogue: into L2 now, so that the
                    // consumers' loads do not wait behind the weight stream in the memory queues
                    const int rows_all = slot_rows<GU>(p, sh);
#pragma unroll
                    for (int m = 0; m < C::kMats; ++m) {
                        const float *sc = GU ? (m ? (sh ? p.wt.sh_u_scale : p.wt.u_scale) : (sh ? p.wt.sh_g_scale : p.wt.g_scale))
                                             : (sh ? p.wt.sh_d_scale : p.wt.d_scale);
                        const float *row = sc + (size_t)ez * rows_all + it.row0;
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(row));
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(row + 32));
                    }
                }
                const int nst = (Kb + C::kStageK - 1) / C::kStageK;
                // decode variant: token rows of the B operand, copied stage by stage
                const unsigned char *brows[8];
                int nb = 0;
                if constexpr (C::kSmemB) {
                    const bool perm_b = GU && FMT == MOE_FMT_INT4_ROWSCALE && (i < n_pre || !p.xb_perm);
                    nb = min(it.ntok, 8);
                    for (int j = 0; j < 8; ++j) {
                        if (C::kLimbs) brows[j] = j < nb ? item_brow_limbs<GU>(p, it, j) : nullptr;
                        else brows[j] = j < nb ? reinterpret_cast<const unsigned char *>(item_brow<GU>(p, it, j, perm_b)) : nullptr;
                    }
                }
                // bytes of a B row that stage s needs, and where they start
                // (limb rows end at their last 256-value block: an int2 stage's second block
                // may lie past it)
                auto b_src = [&](int s2) -> size_t { return C::kLimbs ? (size_t)s2 * C::kBRow : (size_t)4 * s2 * C::kStageK; };
                auto b_len = [&](int s2) -> uint32_t {
                    return C::kLimbs ? (uint32_t)min((size_t)C::kBRow, limb_row_bytes(it.K) - (size_t)s2 * C::kBRow)
                                     : 4u * (uint32_t)min(C::kStageK, Kb - s2 * C::kStageK);
                };
                // The down kernel starts early (programmatic launch) and its B operand, h,
                // comes from the gate/up kernel: its first stages get their weights at once
                // and their h rows only after the grid dependency is resolved.
                const int defer = ((!GU || C::kLimbs) && C::kSmemB && !pdl_done) ? min(nst, S) : 0;
                for (int s = 0; s < nst; ++s) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) { ok = false; break; }
                    unconfirmed &= ~(1u << stage);
                    const int kb0 = s * C::kStageK;
                    // K boxes of this stage (KS for the K-split launches, two for int8)
                    const int nks = min(KS * C::kBoxesK, (Kb - kb0 + kBoxBytes - 1) / kBoxBytes);
                    const uint32_t bbytes = b_len(s);
                    uint32_t tx = (uint32_t)C::kMats * RW * nks * (kBoxSmem + (C::kNv ? kScaleBoxSmem : 0));
                    if constexpr (C::kSmemB) {
                        for (int j = 0; j < nb; ++j) tx += brows[j] ? bbytes : 0u;
                    }
                    mbar_arrive_expect_tx(&full[stage], tx);
                    unsigned char *st = ring + (size_t)stage * C::kStageBytes;
#pragma unroll
                    for (int m = 0; m < C::kMats; ++m) {
                        const CUtensorMap *map = sh ? (m ? mS1 : mS0) : (m ? mA1 : mA0);
                        const CUtensorMap *bm = sh ? (m ? bS1 : bS0) : (m ? bA1 : bA0);
                        for (int rw = 0; rw < (kBox64 ? 1 : RW); ++rw)
                            for (int ks = 0; ks < nks; ++ks) {
                                // (a 64-row box lands as the four 16-row boxes, stacked;
                                // int8's second K box follows the first)
                                const int bx = rw * KS + ks;
                                unsigned char *dst = C::kBoxesK > 1 ? st + m * C::kMatBytes + ks * kMatStage
                                                                    : st + m * kMatStage + bx * kBoxSmem;
                                tma_load_3d(dst, map, &full[stage], kb0 + ks * kBoxBytes, it.row0 + rw * kRowTile,
                                            ez, pol);
                                if (C::kNv)
                                    tma_load_3d(st + C::kCodeBytes + (m * kConsumerWarps + bx) * kScaleBoxSmem, bm,
                                                &full[stage], (kb0 + ks * kBoxBytes) / 8, it.row0 + rw * kRowTile,
                                                ez, pol);
                            }
                    }
                    if constexpr (C::kSmemB) {
                        if (s >= defer) {
                            for (int j = 0; j < nb; ++j)
                                if (brows[j])
                                    bulk_copy(bring + (size_t)stage * p.b_stage + j * C::kBRow, brows[j] + b_src(s), bbytes,
                                              &full[stage]);
                        }
                        if (defer && s == defer - 1) {
                            // h (x limbs) is complete once the gate/up grid (router) is:
                            // the deferred rows now
                            pdl_wait();
                            pdl_done = true;
                            int st2 = stage - (defer - 1);
                            if (st2 < 0) st2 += S;
                            for (int s2 = 0; s2 < defer; ++s2) {
                                for (int j = 0; j < nb; ++j)
                                    if (brows[j])
                                        bulk_copy(bring + (size_t)st2 * p.b_stage + j * C::kBRow, brows[j] + b_src(s2),
                                                  b_len(s2), &full[st2]);
                                if (++st2 == S) st2 = 0;
                            }
                        }
                    }
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    unconfirmed |= 1u << stage;
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) *abort_flag = 1;
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (*abort_flag) ok = false;
        }
        if (!have_table && lane == 0) mbar_arrive(table_ready);  // release the consumers (never waited for)
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
    L.rw = warp / KS;
    L.ks = warp % KS;
    L.bx = L.rw * KS + L.ks;
    L.dk = p.dk;
    {
        // ldmatrix: lane -> (row inside the 16-row box, first or second chunk of a pair)
        const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int lch = lane >> 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) L.off[q] = lrow * kBoxBytes + ((((2 * q + lch) ^ (lrow & 7)) & 7) << 4);
    }
    int stage = 0;
    uint32_t phase = 0;
    bool have_table = false;
    int total = n_pre;
    Pending pend;
    pend.kind = 0;

    // cfail is written only by consumer warps and read only after a consumer barrier,
    // so all four warps take the same exit decision and meet at the same barriers.
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
        if (i >= n_pre && !have_table) {
            if (!mbar_wait(table_ready, 0, p.status)) {
                *cfail = 1;
                *abort_flag = 1;
            }
            consumer_sync();
            if (*cfail) break;
            have_table = true;
            total = tb.hdr[1];
            if (GU) {
                pdl_wait();     // topk and the routed buckets come from the router
                pdl_trigger();
            }
        }
        const Item it = (i < n_pre) ? make_item<GU, RW>(p, -1, p.T, 0, i) : decode_item<GU, RW>(p, tb, i);
        const bool sh = it.e < 0;
        const uint32_t zsm = smem_u32(zrow_sm);
        if constexpr (C::kLimbs) {
            // x limbs come from the router, h limbs from the gate/up kernel
            if (n_item == 0) pdl_wait();
            const bool ok = it.ntok <= 2
                                ? consume_item_limbs<FMT, GU, 1>(p, tb, it, ring, bring, full, empty, stage, phase, L,
                                                                 zsm, pend, cfail, abort_flag)
                                : consume_item_limbs<FMT, GU, 3>(p, tb, it, ring, bring, full, empty, stage, phase, L,
                                                                 zsm, pend, cfail, abort_flag);
            if (!ok) break;
            continue;
        } else {

        // B-operand rows of this thread's tokens (one per n-tile: column 8n + g); padding
        // columns read a zero row, so no lane needs a select in the inner loop
        const bool perm_b = GU && FMT == MOE_FMT_INT4_ROWSCALE && (i < n_pre || !p.xb_perm);
        BRows brow;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int col = 8 * n + L.g;
            brow.r[n] = p.zrow;
            if (col < it.ntok) {
                const int bpos = it.tok0 + col;
                if (GU) {
                    int t = bpos;
                    if (!sh) {
                        const int a = __ldg(p.perm + it.boff + bpos);
                        t = (a >= 0 && a < p.T * p.k) ? a / p.k : -1;
                        if (t < 0) record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                    }
                    if (t >= 0) brow.r[n] = (perm_b ? p.x : p.xb) + (size_t)t * p.H;
                } else {
                    brow.r[n] = sh ? reinterpret_cast<const uint16_t *>(p.h_sh) + (size_t)bpos * p.I_sh
                                 : reinterpret_cast<const uint16_t *>(p.h) + (size_t)(it.boff + bpos) * p.I;
                }
            }
        }
        if (!GU && n_item == 0) pdl_wait();   // h is produced by the gate/up kernel

        const int nN = (it.ntok + 7) >> 3;
        bool ok;
        constexpr bool kPerm = GU && FMT == MOE_FMT_INT4_ROWSCALE;
#define MOE_CONSUME(NN, PERM)                                                                                   \
    consume_item<FMT, GU, KS, NNMAX, NN, PERM>(p, tb, it, ring, bring, full, empty, stage, phase, L, brow, zsm, red, \
                                               cfail, abort_flag)
        // NNMAX = 1: items of at most 8 tokens (decode), one n-tile, few registers.
        // NNMAX = 4: items of up to 32 tokens; 2 and 3 n-tiles run the 4-tile code
        // (padding columns read the zero row), which keeps the kernel small.
        if constexpr (NNMAX == 1) {
            if (kPerm && perm_b) ok = MOE_CONSUME(1, kPerm);
            else ok = MOE_CONSUME(1, false);
        } else {
            if (kPerm && perm_b) ok = nN == 1 ? MOE_CONSUME(1, kPerm) : MOE_CONSUME(4, kPerm);
            else ok = nN == 1 ? MOE_CONSUME(1, false) : MOE_CONSUME(4, false);
        }
#undef MOE_CONSUME
        if (!ok) break;
        }
    }
    if constexpr (C::kLimbs && GU) {
        // the last item's completion check (all consumer warps arrive here together, so
        // the barriers inside line up; a failed CTA has nothing pending to settle safely)
        if (!*cfail) settle<GU>(p, pend, threadIdx.x);
    }
    // the last CTA to finish resets the work counters (every producer has made its last
    // claim before its consumers saw the end of the queue)
    if (tid == 0 && !*cfail && atomicAdd(p.work + 1, 1u) == (unsigned)G - 1u) {
        atomicExch(p.work, 0u);
        atomicExch(p.work + 1, 0u);
    }
}

// ============================================================================ tcgen05 path
// Expert GEMMs of larger batches (int4, T > 16): each work item is (expert, 128 output
// rows, up to kTcTok tokens).  Arithmetic as on the decode path: weights as s8 bytes
// 16 x code, activations as three exact int8 limbs, exact integer accumulation; here the
// product runs on the 5th-generation tensor cores (tcgen05.mma kind::i8, M = 128,
// N = 3 x tokens rounded up to 16, K = 32 per instruction, s32 accumulators in TMEM).
//
// Warps: 0 streams the packed codes with TMA into a ring of 256-K stages; 1 allocates
// TMEM and issues the MMAs (one thread); 2..9 expand each 128-K half of a stage to int8
// and store it straight into tensor memory, where the MMA reads its A operand (row r =
// TMEM lane r, four s8 per column), and copy the tokens' limb rows for that half into a
// ring of shared-memory B slots (asynchronous 16-byte copies, in the 128-byte-swizzled
// K-major layout, several halves ahead); 10..13 read an item's accumulators from TMEM
// once they are complete (warp w owns TMEM lanes 32 (w % 4) ..) and run the epilogue.
// With the expanded weights in TMEM, shared memory carries only the packed codes (one
// TMA write, one read: a quarter of the bytes an expanded s8 tile would move twice) and
// the B slots.  Accumulators are double-buffered in TMEM, so the next item's MMAs overlap
// an epilogue.  One tcgen05.mma of this shape costs about the same for any N up to 256
// and the issuing thread's own instructions add to it, so with ~16-18 tokens per expert
// the kernel is bound by MMA issue, not by MACs.

constexpr int kTcRows = 128;                    // output rows per item (MMA M)
constexpr int kTcTok = 32;                      // tokens per item (batches of few tokens per expert)
constexpr int kTcTokWide = 64;                  // tokens per item when experts average more than 36
constexpr int kTcPackMax = 8;                   // packed stages (256 K each) at most
constexpr int kTcASub = 2;                      // expanded 128-K halves held in TMEM
constexpr int kTcBMax = 8;                      // B slots at most
constexpr int kTcConv = 8;                      // converter warps (two per TMEM lane quarter)
constexpr int kTcConvT = kTcConv * 32;
constexpr int kTcEpi = 4;                       // epilogue warps (one per TMEM lane quarter)
constexpr int kTcThreads = (2 + kTcConv + kTcEpi) * 32;
// dynamic shared memory the kernel may take (the device's opt-in maximum less a margin
// for static shared memory)
constexpr size_t kTcSmemMax = 232448 - 1024;
// TOK tokens per item: N = 3 TOK limb columns at most.  With 64-token items (batches of
// many tokens per expert: each weight byte is read once for twice the tokens, and each MMA
// carries twice the columns) the gate/up accumulators take 384 of the 512 TMEM columns, so
// they are single-buffered there (the next item's MMAs wait for the epilogue).
template <bool GU, int TOK>
struct TcCfg {
    static constexpr int kMats = GU ? 2 : 1;
    static constexpr int kNMax = 3 * TOK;                            // limb columns of an item
    static constexpr int kBSlot = kNMax * 128;                       // one B slot: the limb rows of 128 K
    static constexpr int kPackBytes = kMats * kTcRows * kBoxBytes;   // one 256-K stage of codes
    static constexpr int kAccCols = kMats * kNMax;                   // TMEM columns of one accumulator set
    static constexpr int kACols = kMats * 32;                        // TMEM columns of one expanded 128-K half
    static constexpr int kNAcc = 2 * kAccCols + kTcASub * kACols <= 512 ? 2 : 1;   // accumulator sets
    static constexpr int kACol0 = kNAcc * kAccCols;                  // first A column
    static constexpr int kTmemCols = kACol0 + kTcASub * kACols <= 256 ? 256 : 512;   // (a power of two)
    static constexpr int kBSlots = TOK > kTcTok ? 4 : (GU ? 4 : 6);
    static_assert(kACol0 + kTcASub * kACols <= kTmemCols, "TMEM budget");
    static_assert(kBSlot % 1024 == 0, "B slots keep the 1024-byte swizzle atoms aligned");
    static_assert(kBSlots <= kTcBMax, "B slot barriers");
};

// dynamic shared memory of a launch with np packed stages: stages, B slots, slot table,
// item metadata, barriers
template <bool GU, int TOK>
__host__ __device__ constexpr size_t tc_smem(int E, int np)
{
    using C = TcCfg<GU, TOK>;
    return 1024 + (size_t)np * C::kPackBytes + (size_t)C::kBSlots * C::kBSlot + (size_t)4 * 4 * (E + 2) + 64 +
           2 * TOK * 16 + 8 + 8 + (2 * kTcPackMax + 2 * kTcASub + kTcBMax + 4 + 2 * kItemQ + 1) * 8;
}

// packed stages of a launch: as many as fit (at most kTcPackMax)
template <bool GU, int TOK>
static int tc_pack_stages(int E)
{
    const size_t base = tc_smem<GU, TOK>(E, 0);
    const int n = base < kTcSmemMax ? (int)((kTcSmemMax - base) / TcCfg<GU, TOK>::kPackBytes) : 0;
    return n > kTcPackMax ? kTcPackMax : n;
}

// UMMA shared-memory descriptor of a K-major tile of 8-row x 128-byte swizzle atoms
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// UMMA instruction descriptor: s8 x s8 -> s32, both K-major, M = 128
__device__ __forceinline__ uint32_t umma_idesc_s8(int n)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);
}

// tcgen05.mma kind::i8 (s8 x s8 -> s32), one CTA, A operand in tensor memory, B by descriptor
__device__ __forceinline__ void umma_s8_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
                 "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate));
}

// registers -> 16 consecutive TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
                 "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr));
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

template <bool GU, int TOK>
__global__ void __launch_bounds__(kTcThreads, 1) ffn_tc_kernel(const __grid_constant__ LayerMaps maps, const FfnParams p)
{
    using C = TcCfg<GU, TOK>;
    constexpr int RW = kTcRows / kRowTile;   // 8: items of 128 rows
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *pack = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NP = p.stages;                                                  // packed stages of this launch
    unsigned char *bring = pack + (size_t)NP * C::kPackBytes;                 // B slots (1024-aligned: all sizes are)
    constexpr int NB = C::kBSlots;
    int *tbl = reinterpret_cast<int *>(bring + (size_t)NB * C::kBSlot);
    const int E = p.E;
    SlotTable tb;
    tb.e = tbl;
    tb.cnt = tbl + (E + 2);
    tb.off = tbl + 2 * (E + 2);
    tb.base = tbl + 3 * (E + 2);
    tb.hdr = tbl + 4 * (E + 2);
    volatile int *abort_flag = tb.hdr + 2;
    volatile int *cfail = tb.hdr + 3;
    volatile int *q_item = tb.hdr + 4;
    const unsigned char **s_brow = reinterpret_cast<const unsigned char **>(tb.hdr + 16);   // [2][TOK] limb rows
    float *s_sc = reinterpret_cast<float *>(s_brow + 2 * TOK);   // [2][TOK] activation scale of each token
    int *s_id = reinterpret_cast<int *>(s_sc + 2 * TOK);         // [2][TOK] token (gate/up) or assignment (down)
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(s_id + 2 * TOK);
    uint64_t *bars = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(s_tmem + 2) + 7) & ~uintptr_t(7));
    uint64_t *pk_full = bars, *pk_empty = pk_full + kTcPackMax;
    uint64_t *sb_full = pk_empty + kTcPackMax, *sb_empty = sb_full + kTcASub;   // expanded halves in TMEM
    uint64_t *b_empty = sb_empty + kTcASub;                                     // B slots
    uint64_t *acc_full = b_empty + kTcBMax, *acc_empty = acc_full + 2;
    uint64_t *q_full = acc_empty + 2, *q_empty = q_full + kItemQ;
    uint64_t *table_ready = q_empty + kItemQ;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    if constexpr (!GU) pdl_trigger();   // the combine kernel may start at once: it waits for this grid
    const int n_pre = GU ? shared_items<GU, RW>(p) : 0;

    if (tid == 0) {
        for (int s = 0; s < NP; ++s) {
            mbar_init(&pk_full[s], 1);
            mbar_init(&pk_empty[s], kTcConv);
        }
        for (int s = 0; s < kTcASub; ++s) {
            mbar_init(&sb_full[s], kTcConv);
            mbar_init(&sb_empty[s], 1);
        }
        for (int s = 0; s < NB; ++s) mbar_init(&b_empty[s], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], kTcEpi);
        }
        for (int q = 0; q < kItemQ; ++q) {
            mbar_init(&q_full[q], 1);
            mbar_init(&q_empty[q], 1 + kTcConv + kTcEpi);
        }
        mbar_init(table_ready, 1);
        tb.hdr[2] = 0;
        tb.hdr[3] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(C::kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ======================================================== producer: packed codes
        const CUtensorMap *mA0 = GU ? &maps.g4 : &maps.d4, *mA1 = &maps.u4;
        const CUtensorMap *mS0 = GU ? &maps.sh_g4 : &maps.sh_d4, *mS1 = &maps.sh_u4;
        const uint64_t pol = l2_evict_first_policy();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, have_table = false;
        int total = n_pre;
        uint32_t unconfirmed = 0, issued_phase = 0;
        for (int n_item = 0;; ++n_item) {
            const int i = (int)__shfl_sync(0xffffffffu, lane == 0 ? atomicAdd(p.work, 1u) : 0u, 0);
            if (ok && i >= n_pre && !have_table) {
                if (GU) pdl_wait();   // routing is complete (the down kernel's table sources are older)
                build_slot_table<GU, RW>(p, tb, E);
                if (lane == 0) mbar_arrive(table_ready);
                have_table = true;
                total = tb.hdr[1];
                if (GU) pdl_trigger();
            }
            const bool done = !ok || i >= total;
            if (lane == 0) {
                const int q = n_item % kItemQ;
                if (!mbar_wait(&q_empty[q], (uint32_t)(((n_item / kItemQ) & 1) ^ 1), p.status)) ok = false;
                q_item[q] = done ? -1 : i;
                mbar_arrive(&q_full[q]);
            }
            if (done) break;
            if (lane == 0 && ok) {
                const Item it = (i < n_pre) ? make_item<GU, RW>(p, -1, p.T, 0, i) : decode_item<GU, RW>(p, tb, i);
                const bool sh = it.e < 0;
                const int ez = sh ? 0 : it.e;
                const int nst = (it.K / 2 + kBoxBytes - 1) / kBoxBytes;
                for (int s = 0; s < nst; ++s) {
                    if (!mbar_wait(&pk_empty[stage], phase ^ 1u, p.status)) { ok = false; break; }
                    unconfirmed &= ~(1u << stage);
                    mbar_arrive_expect_tx(&pk_full[stage], (uint32_t)C::kPackBytes);
                    unsigned char *st = pack + (size_t)stage * C::kPackBytes;
#pragma unroll
                    for (int m = 0; m < C::kMats; ++m) {
                        const CUtensorMap *map = sh ? (m ? mS1 : mS0) : (m ? mA1 : mA0);
#pragma unroll
                        for (int h = 0; h < 2; ++h)   // two 64-row boxes
                            tma_load_3d(st + (m * kTcRows + 64 * h) * kBoxBytes, map, &pk_full[stage], s * kBoxBytes,
                                        it.row0 + 64 * h, ez, pol);
                    }
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    unconfirmed |= 1u << stage;
                    if (++stage == NP) { stage = 0; phase ^= 1u; }
                }
                if (!ok) *abort_flag = 1;
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (*abort_flag) ok = false;
        }
        if (!have_table && lane == 0) mbar_arrive(table_ready);
        if (lane == 0 && !ok)
            for (int s = 0; s < NP; ++s)
                if (unconfirmed >> s & 1u) mbar_wait(&pk_full[s], issued_phase >> s & 1u, p.status, 10000000ull);
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        int sub = 0, gs = 0;   // expanded half (TMEM); halves so far (B slot gs % NB)
        uint32_t sphase = 0;
        bool ok = true, have_table = false;
        for (int n_item = 0; ok; ++n_item) {
            const int q = n_item % kItemQ;
            int i = -1;
            if (mbar_wait(&q_full[q], (uint32_t)((n_item / kItemQ) & 1), p.status)) i = q_item[q];
            else ok = false;
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_empty[q]);
            if (i < 0) break;
            if (i >= n_pre && !have_table) {
                if (!mbar_wait(table_ready, 0, p.status)) { ok = false; break; }
                have_table = true;
            }
            const Item it = (i < n_pre) ? make_item<GU, RW>(p, -1, p.T, 0, i) : decode_item<GU, RW>(p, tb, i);
            const int n = ((3 * it.ntok + 15) / 16) * 16;
            const uint32_t idesc = umma_idesc_s8(n);
            const int buf = n_item % C::kNAcc;
            // the epilogue of the item kNAcc back has released this accumulator set
            if (!mbar_wait(&acc_empty[buf], (uint32_t)(((n_item / C::kNAcc) & 1) ^ 1), p.status)) { ok = false; break; }
            tc_fence_after();
            const int nsub = (it.K + 127) / 128;   // 128-K halves of the packed stages
            for (int u = 0; u < nsub; ++u) {
                if (!mbar_wait(&sb_full[sub], sphase, p.status)) { ok = false; break; }
                tc_fence_after();
                const int kvals = min(128, it.K - 128 * u);   // a multiple of 64
                const int bslot = gs % NB;
                if (lane == 0) {
                    // The issuing thread's own instructions between MMAs add to every MMA's
                    // cost (measured), so the operands are formed once per half: the B
                    // descriptor advances 32 bytes (2 in its 16-byte address field) per step.
                    const uint64_t db0 = umma_sdesc(smem_u32(bring + (size_t)bslot * C::kBSlot));
                    const uint32_t abase = tmem + C::kACol0 + sub * C::kACols;
                    const uint32_t dbase = tmem + buf * C::kAccCols;
                    const uint32_t acc0 = u > 0 ? 1u : 0u;
                    if (kvals == 128) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                            for (int m = 0; m < C::kMats; ++m)
                                umma_s8_ta(dbase + m * C::kNMax, abase + m * 32 + 8 * kk, db0 + 2 * kk, idesc,
                                           kk > 0 ? 1u : acc0);
                    } else {
                        for (int kk = 0; kk < kvals / 32; ++kk)
#pragma unroll
                            for (int m = 0; m < C::kMats; ++m)
                                umma_s8_ta(dbase + m * C::kNMax, abase + m * 32 + 8 * kk, db0 + 2 * kk, idesc,
                                           kk > 0 ? 1u : acc0);
                    }
                    umma_commit(&sb_empty[sub]);   // the half and the B slot are free once
                    umma_commit(&b_empty[bslot]);  // these MMAs have read them
                    if (u == nsub - 1) umma_commit(&acc_full[buf]);
                }
                __syncwarp();
                ++gs;
                if (++sub == kTcASub) { sub = 0; sphase ^= 1u; }
            }
        }
        if (!ok) *abort_flag = 1;
    } else {
        // ======================================================== converters / epilogue
        // the item sequence, as the producer announces it (every role reads it)
        auto next_item = [&](int n_item, int &i) -> bool {
            const int q = n_item % kItemQ;
            i = -1;
            const bool got = mbar_wait(&q_full[q], (uint32_t)((n_item / kItemQ) & 1), p.status);
            if (got) i = q_item[q];
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_empty[q]);
            return got;
        };
        if (warp < 2 + kTcConv) {
            // -------------------------------------------------------- converters
            const int ltid = tid - 64;   // 0 .. kTcConvT - 1
            int pstage = 0, sub = 0, gsub = 0;   // gsub: halves of earlier items (B slots used)
            uint32_t pphase = 0, sphase = 0;
            bool have_table = false;
            for (int n_item = 0;; ++n_item) {
                int i;
                if (!next_item(n_item, i)) {
                    *cfail = 1;
                    *abort_flag = 1;
                }
                consumer_sync<kTcConvT, 1>();
                if (*cfail || i < 0) break;
                if (i >= n_pre && !have_table) {
                    if (!mbar_wait(table_ready, 0, p.status)) {
                        *cfail = 1;
                        *abort_flag = 1;
                    }
                    consumer_sync<kTcConvT, 1>();
                    if (*cfail) break;
                    have_table = true;
                }
                if (n_item == 0) pdl_wait();   // limb rows come from the router / the gate/up kernel
                const Item it = (i < n_pre) ? make_item<GU, RW>(p, -1, p.T, 0, i) : decode_item<GU, RW>(p, tb, i);
                const int nrow = 3 * it.ntok;
                // the item's limb rows (one per token)
                if (ltid < it.ntok) s_brow[ltid] = item_brow_limbs<GU>(p, it, ltid);
                consumer_sync<kTcConvT, 1>();
                const int nst = (it.K / 2 + kBoxBytes - 1) / kBoxBytes;
                const int nsub = (it.K + 127) / 128;
                // B: the 3 x tokens limb rows of every 128-K half, 16-byte pieces (8 per row),
                // copied into B slot (gsub + half) % NB in the swizzled layout the MMA reads, up
                // to NB - 2 halves ahead (a slot is refilled two halves after its last use, so the
                // copies never wait for the MMAs just handed over).  Thread ltid owns pieces
                // ltid + 256 q of each half.
                constexpr int NQ = 3 * TOK * 8 / kTcConvT;
                const unsigned char *bsrc[NQ];
                int bdst[NQ];
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    const int pc = ltid + q * kTcConvT, jr = pc >> 3, x = pc & 7;
                    bsrc[q] = nullptr;
                    bdst[q] = -1;
                    if (jr < nrow) {
                        bdst[q] = jr * 128 + ((x ^ (jr & 7)) << 4);
                        const unsigned char *br = s_brow[jr / 3];
                        if (br) bsrc[q] = br + (jr % 3) * kLimbBlockK + 16 * x;
                    }
                }
                const int ahead = min(NB - 2, nsub);
                bool ok = true;
                auto bissue = [&](int u2) {   // half u2 of this item into its slot (one commit group)
                    const int g = gsub + u2, slot = g % NB;
                    if (!mbar_wait(&b_empty[slot], (uint32_t)(((g / NB) & 1) ^ 1), p.status)) ok = false;
                    if (ok) {
                        unsigned char *sl = bring + (size_t)slot * C::kBSlot;
                        const size_t so = (size_t)(u2 >> 1) * kLimbBlockBytes + 128 * (u2 & 1);
#pragma unroll
                        for (int q = 0; q < NQ; ++q) {
                            if (bdst[q] < 0) continue;
                            if (bsrc[q]) cp_async16(sl + bdst[q], bsrc[q] + so);
                            else *reinterpret_cast<uint4 *>(sl + bdst[q]) = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    cp_async_commit();
                };
                for (int u2 = 0; u2 < ahead; ++u2) bissue(u2);
                // A: this thread expands row r of matrix m (gate/up), or one 64-K group of row r
                // (down: the two warps of a lane quarter split each half), into TMEM lane r
                const int cw = warp - 2, quarter = warp & 3, r = 32 * quarter + lane;
                const int m = GU ? cw / 4 : 0, g0 = GU ? 0 : cw / 4, ng = GU ? 2 : 1;
                const uint32_t tlane = tmem + ((uint32_t)(32 * quarter) << 16);
                for (int s = 0; s < nst && ok; ++s) {
                    if (!mbar_wait(&pk_full[pstage], pphase, p.status)) { ok = false; break; }
                    const unsigned char *prow = pack + (size_t)pstage * C::kPackBytes + (size_t)(m * kTcRows + r) * kBoxBytes;
                    for (int u = 0; u < 2; ++u) {
                        const int k0 = 256 * s + 128 * u;   // first K value of this half
                        if (k0 >= it.K) break;
                        if (!mbar_wait(&sb_empty[sub], sphase ^ 1u, p.status)) { ok = false; break; }
                        tc_fence_after();
                        // packed row bytes [64u, 64u + 64) -> 128 s8 bytes in limb order: 64-K group
                        // gq -> columns 16 gq .. 16 gq + 15 of the half (words tq, tq + 4 of the group
                        // -> columns 4 tq .. 4 tq + 3: their even, then their odd elements)
                        for (int gi = 0; gi < ng; ++gi) {
                            const int gq = g0 + gi;
                            const int c0 = 4 * u + 2 * gq;   // packed chunks c0 (words 0-3), c0 + 1 (words 4-7)
                            const uint4 lo = *reinterpret_cast<const uint4 *>(prow + ((c0 ^ (r & 7)) << 4));
                            const uint4 hi = *reinterpret_cast<const uint4 *>(prow + (((c0 + 1) ^ (r & 7)) << 4));
                            const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
                            uint32_t v[16];
#pragma unroll
                            for (int tq = 0; tq < 4; ++tq) {
                                int4_word_to_s8x16(wl[tq], v[4 * tq], v[4 * tq + 2]);
                                int4_word_to_s8x16(wh[tq], v[4 * tq + 1], v[4 * tq + 3]);
                            }
                            tmem_st16(tlane + C::kACol0 + sub * C::kACols + m * 32 + 16 * gq, v);
                        }
                        // the B copies of a later half, then wait for this half's
                        const int uu = 2 * s + u;
                        if (uu + ahead < nsub) bissue(uu + ahead);
                        else cp_async_commit();
                        cp_async_wait_n(ahead);
                        tmem_wait_st();
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // B visible to the tensor cores
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sb_full[sub]);
                        if (++sub == kTcASub) { sub = 0; sphase ^= 1u; }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pk_empty[pstage]);
                    if (++pstage == NP) { pstage = 0; pphase ^= 1u; }
                }
                gsub += nsub;
                if (!ok) {
                    *cfail = 1;
                    *abort_flag = 1;
                }
            }
        } else {
            // -------------------------------------------------------- epilogue
            const int etid = tid - 64 - kTcConvT;   // 0..127
            const int quarter = warp & 3;           // TMEM lane quarter this warp may access
            const int row_l = 32 * quarter + lane;  // the output row (TMEM lane) of this thread
            bool have_table = false, ok = true;
            Pending pend;
            pend.kind = 0;
            for (int n_item = 0;; ++n_item) {
                int i;
                if (!next_item(n_item, i)) ok = false;
                if (!ok || i < 0) break;
                if (i >= n_pre && !have_table) {
                    if (!mbar_wait(table_ready, 0, p.status)) { ok = false; break; }
                    have_table = true;
                }
                if (n_item == 0) pdl_wait();
                const Item it = (i < n_pre) ? make_item<GU, RW>(p, -1, p.T, 0, i) : decode_item<GU, RW>(p, tb, i);
                const bool sh = it.e < 0;
                // the item's tokens: activation scales and ids, loaded while the MMAs run
                if (etid < it.ntok) {
                    const int bpos = it.tok0 + etid;
                    int id = bpos;     // shared expert: the token itself
                    if (!sh) {
                        const int aid = __ldg(p.perm + it.boff + bpos);
                        id = (aid >= 0 && aid < p.T * p.k) ? (GU ? aid / p.k : aid) : -1;
                    }
                    s_id[etid] = id;
                    s_sc[etid] = GU ? (id >= 0 ? __ldcg(p.x_limb_scale + id) : 0.f)
                                    : __ldcg(sh ? p.hsh_limb_scale + bpos : p.h_limb_scale + it.boff + bpos);
                }
                consumer_sync<kTcConvT / 2, 2>();
                const int buf = n_item % C::kNAcc;
                if (!mbar_wait(&acc_full[buf], (uint32_t)((n_item / C::kNAcc) & 1), p.status)) { ok = false; break; }
                tc_fence_after();
                const int rows_all = slot_rows<GU>(p, sh);
                const int ez = sh ? 0 : it.e;
                const int row = it.row0 + row_l;
                const float *sc0 = GU ? (sh ? p.wt.sh_g_scale : p.wt.g_scale) : (sh ? p.wt.sh_d_scale : p.wt.d_scale);
                const float *sc1 = sh ? p.wt.sh_u_scale : p.wt.u_scale;
                const double rs0 = (double)__ldg(sc0 + (size_t)ez * rows_all + row);
                const double rs1 = GU ? (double)__ldg(sc1 + (size_t)ez * rows_all + row) : 0.0;
                const uint32_t tbase = tmem + ((uint32_t)(32 * quarter) << 16) + buf * C::kAccCols;
                const float *msc = s_sc;
                const int *mid = s_id;
                for (int j0 = 0; j0 < it.ntok; j0 += 8) {   // 8 tokens = 24 accumulator columns per matrix
                    uint32_t a[C::kMats][24];
#pragma unroll
                    for (int m = 0; m < C::kMats; ++m)
#pragma unroll
                        for (int c8 = 0; c8 < 3; ++c8) {
                            uint32_t v[8];
                            tmem_ld8(tbase + m * C::kNMax + 3 * j0 + 8 * c8, v);
#pragma unroll
                            for (int x = 0; x < 8; ++x) a[m][8 * c8 + x] = v[x];
                        }
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        const int j = j0 + jj;
                        const bool valid = j < it.ntok;
                        long long Sv[C::kMats];
#pragma unroll
                        for (int m = 0; m < C::kMats; ++m)
                            Sv[m] = (long long)((int)a[m][3 * jj] >> 4) + 256ll * ((int)a[m][3 * jj + 1] >> 4) +
                                    65536ll * ((int)a[m][3 * jj + 2] >> 4);
                        const int bpos = it.tok0 + j;
                        if (GU) {
                            float hm = 0.f;
                            if (valid) {
                                float hv = 0.f;
                                const int tok = mid[j];
                                if (tok < 0) record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                                else {
                                    const double xs = (double)msc[j];
                                    const float gv = (float)((double)Sv[0] * xs * rs0);
                                    const float uv = (float)((double)Sv[C::kMats - 1] * xs * rs1);
                                    hv = gv / (1.f + expf(-gv)) * uv;
                                }
                                __half *dst = sh ? p.h_sh + (size_t)bpos * p.I_sh : p.h + (size_t)(it.boff + bpos) * p.I;
                                const __half hh = __float2half_rn(hv);
                                dst[row] = hh;
                                hm = fabsf(__half2float(hh));
                            }
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) hm = fmaxf(hm, __shfl_xor_sync(0xffffffffu, hm, o));
                            if (valid && lane == 0)
                                atomicMax(p.h_amax + (sh ? p.T * p.k : it.boff) + bpos, __float_as_uint(hm));
                        } else if (valid) {
                            const float yv = (float)((double)Sv[0] * (double)msc[j] * rs0);
                            if (sh) {
                                p.y_shared[(size_t)bpos * p.H + row] = yv;
                            } else {
                                const int aid = mid[j];
                                if (aid >= 0) p.y_assign[(size_t)aid * p.H + row] = yv;
                                else record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
                consumer_sync<kTcConvT / 2, 2>();   // s_sc / s_id are rewritten for the next item
                if (GU) {
                    // the previous item's h conversion (if it completed a token group), then
                    // count this row tile of the group; the last one converts its h rows
                    settle<GU, kTcConvT / 2, 2>(p, pend, etid);
                    consumer_sync<kTcConvT / 2, 2>();
                    pend.kind = 1;
                    pend.sh = sh;
                    pend.tok0 = it.tok0;
                    pend.ntok = it.ntok;
                    pend.boff = it.boff;
                    pend.target = (unsigned)(rows_all / kTcRows) - 1u;
                    if (etid == 0)
                        pend.old = atom_inc_acq_rel(p.chunk_counters + (sh ? p.T * p.k + it.tok0 : it.boff + it.tok0), pend.target);
                }
            }
            if (!ok) {
                *cfail = 1;
                *abort_flag = 1;
            }
            if (GU && ok) settle<GU, kTcConvT / 2, 2>(p, pend, etid);
            if (etid == 0 && ok && atomicAdd(p.work + 1, 1u) == (unsigned)G - 1u) {
                atomicExch(p.work, 0u);
                atomicExch(p.work + 1, 0u);
            }
        }
    }
    // every role is done: release the tensor memory
    cp_async_wait<0>();   // no B copy may still be landing
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols));
    }
}

// ---------------------------------------------------------------------------- test hook
__global__ void wait_timeout_kernel(int *status, unsigned long long max_iters)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, status, 50000000ull /*50 ms*/, max_iters);
}

// ---------------------------------------------------------------------------- launchers
// dynamic shared memory a CTA may use so that two fit on one SM (228 KB, 1 KB reserved
// and up to 1 KB of static shared memory per CTA)
constexpr size_t kSmemPerCta2 = 112 * 1024;
constexpr size_t kSmemPerCta3 = 73 * 1024;   // three CTAs per SM (the int8-path down kernels)

// Ring geometry of a launch: the int8 path stages the B rows of min(T, 8) tokens per
// stage and takes as many stages as fit beside a second CTA (at most its cap).
template <int FMT, bool GU, int KS, int NNMAX>
static void ffn_geometry(int E, int T, int &stages, int &b_stage)
{
    using C = FfnCfg<FMT, GU, KS, NNMAX>;
    if constexpr (C::kLimbs) {
        b_stage = (T < 8 ? (T < 1 ? 1 : T) : 8) * C::kBRow;
        const size_t fixed = ffn_smem<FMT, GU, KS, NNMAX>(E, 0, 0);
        const size_t budget = ffn_min_ctas<FMT, GU, KS, NNMAX>() == 3 ? kSmemPerCta3 : kSmemPerCta2;
        int n = fixed < budget ? (int)((budget - fixed) / (C::kStageBytes + b_stage)) : 0;
        stages = n < 2 ? 2 : (n > C::kStagesCap ? C::kStagesCap : n);
    } else {
        stages = C::kStages;
        b_stage = C::kBBytes;
    }
}

template <int FMT, bool GU, int KS, int NNMAX>
static cudaError_t launch_t(const LayerMaps &maps, const FfnParams &p0, int grid, bool pdl, cudaStream_t s)
{
    // the int8-path variants read the activation limbs: never launch one without them
    if (FfnCfg<FMT, GU, KS, NNMAX>::kLimbs && (!p0.limbs || !p0.x_limbs || !p0.x_limb_scale || !p0.h_limbs ||
                                               !p0.h_limb_scale || !p0.chunk_counters || !p0.h_amax))
        return cudaErrorInvalidValue;
    FfnParams p = p0;
    ffn_geometry<FMT, GU, KS, NNMAX>(p.E, p.T, p.stages, p.b_stage);
    p.work = p0.work + (GU ? 0 : 2);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kFfnThreads);
    cfg.dynamicSmemBytes = ffn_smem<FMT, GU, KS, NNMAX>(p.E, p.stages, p.b_stage);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, ffn_kernel<FMT, GU, KS, NNMAX>, maps, p);
}

template <int FMT, bool GU, int KS, int NNMAX>
static cudaError_t prepare_t(int E, int *blocks_per_sm)
{
    // the limit is a property of the kernel, shared by every handle: the device maximum;
    // the occupancy is that of this handle's largest launch
    size_t smem = 0;
    for (int T = 1; T <= 8; ++T) {
        int st, bs;
        ffn_geometry<FMT, GU, KS, NNMAX>(E, T, st, bs);
        const size_t v = ffn_smem<FMT, GU, KS, NNMAX>(E, st, bs);
        smem = v > smem ? v : smem;
    }
    int dev = 0, optin = 0;
    cudaFuncAttributes fa;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, ffn_kernel<FMT, GU, KS, NNMAX>);
    if (e != cudaSuccess) return e;
    if (smem + fa.sharedSizeBytes > (size_t)optin) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(ffn_kernel<FMT, GU, KS, NNMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - (int)fa.sharedSizeBytes);
    if (e != cudaSuccess) return e;
    // the largest shared-memory carveout, so that the occupancy below is reached and CTAs
    // of the next kernel can start beside this one's
    e = cudaFuncSetAttribute(ffn_kernel<FMT, GU, KS, NNMAX>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, ffn_kernel<FMT, GU, KS, NNMAX>, kFfnThreads,
                                                         smem);
}

// Sets the shared-memory limits of the expert kernels of a format and returns their
// resident CTAs per SM: occ[nnmax == 4][gate_up][ks == 4].
template <int FMT>
static cudaError_t prepare_fmt(int E, int occ[2][2][2])
{
    cudaError_t e;
    if ((e = prepare_t<FMT, true, 1, 1>(E, &occ[0][1][0])) != cudaSuccess) return e;
    if ((e = prepare_t<FMT, false, 1, 1>(E, &occ[0][0][0])) != cudaSuccess) return e;
    if constexpr (FMT == MOE_FMT_INT8_ROWSCALE || FMT == MOE_FMT_INT2_ROWSCALE) {
        // int8 and int2 run the int8 path only (8-token items, KS = 1, any batch)
        for (int w = 0; w < 2; ++w)
            for (int g = 0; g < 2; ++g) occ[w][g][0] = occ[w][g][1] = occ[0][g][0];
        return cudaSuccess;
    } else {
        if constexpr (FMT == MOE_FMT_INT4_ROWSCALE) {
            // the int8 path (int4, items of <= 8 tokens) has no K-split variant
            occ[0][1][1] = occ[0][1][0];
            occ[0][0][1] = occ[0][0][0];
        } else {
            if ((e = prepare_t<FMT, true, 4, 1>(E, &occ[0][1][1])) != cudaSuccess) return e;
            if ((e = prepare_t<FMT, false, 4, 1>(E, &occ[0][0][1])) != cudaSuccess) return e;
        }
        if ((e = prepare_t<FMT, true, 1, 4>(E, &occ[1][1][0])) != cudaSuccess) return e;
        if ((e = prepare_t<FMT, true, 4, 4>(E, &occ[1][1][1])) != cudaSuccess) return e;
        if ((e = prepare_t<FMT, false, 1, 4>(E, &occ[1][0][0])) != cudaSuccess) return e;
        return prepare_t<FMT, false, 4, 4>(E, &occ[1][0][1]);
    }
}

template <bool GU, int TOK>
static cudaError_t tc_prepare_t(int E)
{
    int dev = 0, optin = 0;
    cudaFuncAttributes fa;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, ffn_tc_kernel<GU, TOK>);
    if (e != cudaSuccess) return e;
    if (tc_pack_stages<GU, TOK>(E) < 2 || tc_smem<GU, TOK>(E, tc_pack_stages<GU, TOK>(E)) + fa.sharedSizeBytes > (size_t)optin)
        return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(ffn_tc_kernel<GU, TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - (int)fa.sharedSizeBytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(ffn_tc_kernel<GU, TOK>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

cudaError_t tc_prepare(int E)
{
    cudaError_t e = tc_prepare_t<true, kTcTok>(E);
    if (e == cudaSuccess) e = tc_prepare_t<false, kTcTok>(E);
    if (e == cudaSuccess) e = tc_prepare_t<true, kTcTokWide>(E);
    return e != cudaSuccess ? e : tc_prepare_t<false, kTcTokWide>(E);
}

template <bool GU, int TOK>
static cudaError_t launch_tc_t(const LayerMaps &maps, const FfnParams &p0, int grid, bool pdl, cudaStream_t s)
{
    FfnParams p = p0;
    p.tok_chunk = TOK;
    p.work = p0.work + (GU ? 0 : 2);
    p.stages = tc_pack_stages<GU, TOK>(p.E);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = tc_smem<GU, TOK>(p.E, p.stages);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, ffn_tc_kernel<GU, TOK>, maps, p);
}

// tokens per item of the tensor-memory kernel: 64 when the routed experts average more
// than 36 tokens each (T k / E), else 32
int tc_tokens(const FfnParams &p) { return (long)p.T * p.k > 36l * p.E ? kTcTokWide : kTcTok; }

// One CTA per SM (the kernel takes most of the shared memory and all of the TMEM).
cudaError_t launch_tc(const LayerMaps &maps, const FfnParams &p, bool gate_up, int grid, bool pdl, cudaStream_t s)
{
    if (tc_tokens(p) == kTcTokWide)
        return gate_up ? launch_tc_t<true, kTcTokWide>(maps, p, grid, pdl, s)
                       : launch_tc_t<false, kTcTokWide>(maps, p, grid, pdl, s);
    return gate_up ? launch_tc_t<true, kTcTok>(maps, p, grid, pdl, s) : launch_tc_t<false, kTcTok>(maps, p, grid, pdl, s);
}

cudaError_t ffn_prepare(int fmt, int E, int occ[2][2][2])
{
    switch (fmt) {
    case MOE_FMT_NVFP4: return prepare_fmt<MOE_FMT_NVFP4>(E, occ);
    case MOE_FMT_INT8_ROWSCALE: return prepare_fmt<MOE_FMT_INT8_ROWSCALE>(E, occ);
    case MOE_FMT_INT2_ROWSCALE: return prepare_fmt<MOE_FMT_INT2_ROWSCALE>(E, occ);
    default: return prepare_fmt<MOE_FMT_INT4_ROWSCALE>(E, occ);
    }
}

template <int FMT>
static cudaError_t launch_fmt(const LayerMaps &maps, const FfnParams &p, bool gu, int ks, int grid, bool pdl,
                              cudaStream_t s)
{
    if constexpr (FMT == MOE_FMT_INT8_ROWSCALE || FMT == MOE_FMT_INT2_ROWSCALE) {
        if (p.tok_chunk != 8 || ks != 1) return cudaErrorInvalidValue;
        return gu ? launch_t<FMT, true, 1, 1>(maps, p, grid, pdl, s) : launch_t<FMT, false, 1, 1>(maps, p, grid, pdl, s);
    } else {
        const bool wide = p.tok_chunk > 8;
        if (!wide && (ks == 1 || FMT == MOE_FMT_INT4_ROWSCALE))
            return gu ? launch_t<FMT, true, 1, 1>(maps, p, grid, pdl, s) : launch_t<FMT, false, 1, 1>(maps, p, grid, pdl, s);
        if (!wide) {
            if constexpr (FMT != MOE_FMT_INT4_ROWSCALE)
                return gu ? launch_t<FMT, true, 4, 1>(maps, p, grid, pdl, s) : launch_t<FMT, false, 4, 1>(maps, p, grid, pdl, s);
        }
        if (gu)
            return ks == 1 ? launch_t<FMT, true, 1, 4>(maps, p, grid, pdl, s) : launch_t<FMT, true, 4, 4>(maps, p, grid, pdl, s);
        return ks == 1 ? launch_t<FMT, false, 1, 4>(maps, p, grid, pdl, s) : launch_t<FMT, false, 4, 4>(maps, p, grid, pdl, s);
    }
}

// p.tok_chunk (8 or 32) selects the kernel variant: 8-token items for decode batches,
// 32-token items otherwise.
cudaError_t launch_ffn(const LayerMaps &maps, const FfnParams &p, bool gate_up, int ks, int grid, bool pdl,
                       cudaStream_t s)
{
    switch (p.fmt) {
    case MOE_FMT_NVFP4: return launch_fmt<MOE_FMT_NVFP4>(maps, p, gate_up, ks, grid, pdl, s);
    case MOE_FMT_INT8_ROWSCALE: return launch_fmt<MOE_FMT_INT8_ROWSCALE>(maps, p, gate_up, ks, grid, pdl, s);
    case MOE_FMT_INT2_ROWSCALE: return launch_fmt<MOE_FMT_INT2_ROWSCALE>(maps, p, gate_up, ks, grid, pdl, s);
    default: return launch_fmt<MOE_FMT_INT4_ROWSCALE>(maps, p, gate_up, ks, grid, pdl, s);
    }
}

cudaError_t launch_wait_timeout(int *status, unsigned long long max_iters, cudaStream_t s)
{
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, max_iters);
    return cudaGetLastError();
}

}  // namespace moe
