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
// Design (B200): the weight stream is the whole cost (2 flop per weight per token), so
// every byte is read from HBM exactly once, by TMA, into a ring of shared-memory stages
// (128-byte swizzled 16-row x 128-byte boxes, an L2 evict-first hint), while four
// consumer warps turn the nibbles into fp16 in registers and feed them to mma.sync
// m16n8k16 (the tensor cores are used as a wide dot-product engine: 256 weights per
// instruction, which keeps the issue slots well below the HBM rate; CUDA-core FMA would
// need ~3 instructions per weight and fall behind HBM).  Work items are
// (expert slot, 16 output rows, up to 32 tokens); a persistent grid walks them with a
// fixed stride, so the result does not depend on timing.  Split-K runs across the four
// consumer warps and is reduced in a fixed order through shared memory.
//
// gate/up kernel: h = SiLU(g * sg) * (u * su) rounded to fp16, stored per bucket
//                 position with each 8-column group in mma B-fragment order.
// down kernel:    y_assign[a] = (W_d h) * sd (fp32); with fuse_combine, the last work
//                 item of a 16-row tile also forms y = shared + sum_j w_j y_assign.
//
// Programmatic dependent launch: the gate/up kernel starts the shared expert (which
// needs no routing) before griddepcontrol.wait; the down kernel's producer streams its
// weights before waiting for h.
#include <cuda_fp16.h>
#include <math.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kConsumerWarps = 4;
constexpr int kFfnThreads = (kConsumerWarps + 1) * 32;
constexpr int kBoxBytes = 128;                 // K bytes per TMA box = swizzle span
constexpr int kBoxesPerStage = 2;
constexpr int kStageK = kBoxBytes * kBoxesPerStage;   // 256 bytes (512 weights) of K
constexpr int kBoxSmem = kRowTile * kBoxBytes;        // 2 KB
constexpr int kScaleRowBytes = kStageK / 8;           // NVFP4: one E4M3 per 16 weights
constexpr int kScaleBoxSmem = kRowTile * kScaleRowBytes;   // 512 B
constexpr int kStages = 6;

template <int FMT, bool GU>
struct FfnCfg {
    static constexpr int kMats = GU ? 2 : 1;
    static constexpr bool kNv = FMT == MOE_FMT_NVFP4;
    static constexpr int kCodeBytes = kMats * kBoxesPerStage * kBoxSmem;
    static constexpr int kStageBytes = kCodeBytes + (kNv ? kMats * 1024 : 0);
    static constexpr int kRedFloats = kConsumerWarps * kMats * kTokChunk * kRowTile;
    static constexpr size_t kSmem = 1024 /*align slack*/ + (size_t)kStages * kStageBytes +
                                    (size_t)kRedFloats * 4 + (size_t)4 * (4 * (kMaxExperts + 2)) +
                                    64 + (2 * kStages + 2) * 8;
};

struct SlotTable {
    int *e;      // expert id, -1 = shared expert
    int *cnt;    // tokens in the bucket
    int *off;    // bucket start (position in perm)
    int *base;   // first item of the slot; base[n_slots] = total
    int *hdr;    // [0] = n_slots, [1] = total items
};

struct Item {
    int e;        // expert, -1 = shared
    int row0;     // first output row
    int tok0;     // first bucket position of the chunk (relative to the bucket)
    int ntok;     // tokens in the chunk (1..32)
    int boff;     // bucket start in perm order
    int K;        // input dimension of the matrix
    int rows;
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

template <bool GU>
__device__ __forceinline__ int shared_items(const FfnParams &p)
{
    if (!p.n_shared) return 0;
    return (slot_rows<GU>(p, true) / kRowTile) * ((p.T + kTokChunk - 1) / kTokChunk);
}

// Items of the shared slot are numbered first and need no routing information.
template <bool GU>
__device__ __forceinline__ Item shared_item(const FfnParams &p, int local)
{
    const int rows = slot_rows<GU>(p, true);
    const int tiles = rows / kRowTile;
    Item it;
    it.e = -1;
    it.row0 = (local % tiles) * kRowTile;
    const int chunk = local / tiles;
    it.tok0 = chunk * kTokChunk;
    it.ntok = min(kTokChunk, p.T - it.tok0);
    it.boff = 0;
    it.K = slot_K<GU>(p, true);
    it.rows = rows;
    return it;
}

template <bool GU>
__device__ Item decode_item(const FfnParams &p, const SlotTable &tb, int i)
{
    const int ns = tb.hdr[0];
    int lo = 0, hi = ns - 1;   // last slot with base <= i
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb.base[mid] <= i) lo = mid;
        else hi = mid - 1;
    }
    const int s = lo;
    const bool shared = tb.e[s] < 0;
    const int rows = slot_rows<GU>(p, shared);
    const int tiles = rows / kRowTile;
    const int local = i - tb.base[s];
    Item it;
    it.e = tb.e[s];
    it.row0 = (local % tiles) * kRowTile;
    const int chunk = local / tiles;
    it.tok0 = chunk * kTokChunk;
    it.ntok = min(kTokChunk, tb.cnt[s] - it.tok0);
    it.boff = tb.off[s];
    it.K = slot_K<GU>(p, shared);
    it.rows = rows;
    return it;
}

// Slot table from the expert offsets: the shared expert first, then the non-empty
// experts in ascending order.  Built by one warp.
template <bool GU>
__device__ void build_slot_table(const FfnParams &p, const SlotTable &tb)
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
        acc = shared_items<GU>(p);
    }
    const int rows = slot_rows<GU>(p, false);
    const int tiles = rows / kRowTile;
    for (int eb = 0; eb < p.E; eb += 32) {
        const int e = eb + lane;
        int cnt = 0, off = 0;
        if (e < p.E) {
            off = __ldcg(p.offsets + e);
            cnt = __ldcg(p.offsets + e + 1) - off;
            if (off < 0 || cnt < 0 || off + cnt > p.T * p.k) {   // inconsistent offsets
                record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                cnt = 0;
            }
        }
        const bool has = cnt > 0;
        const unsigned bal = __ballot_sync(0xffffffffu, has);
        const int nit = has ? tiles * ((cnt + kTokChunk - 1) / kTokChunk) : 0;
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

// position of h column n inside its 8-column group, in the order the down kernel's
// B fragments want it (int4: pairs (0,4)(1,5)(2,6)(3,7); NVFP4: natural order)
template <int FMT>
__device__ __forceinline__ int h_pos(int n)
{
    if (FMT == MOE_FMT_NVFP4) return n;
    const int m = n & 7;
    return (n & ~7) | ((m & 3) << 1) | (m >> 2);
}

// named barrier of the four consumer warps (the producer warp never joins it)
__device__ __forceinline__ void consumer_sync()
{
    asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
}

template <int FMT, bool GU>
__global__ void __launch_bounds__(kFfnThreads) ffn_kernel(const __grid_constant__ LayerMaps maps,
                                                          const FfnParams p)
{
    using C = FfnCfg<FMT, GU>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *ring = smem;
    float *red = reinterpret_cast<float *>(ring + (size_t)kStages * C::kStageBytes);
    int *tbl = reinterpret_cast<int *>(red + C::kRedFloats);
    SlotTable tb;
    tb.e = tbl;
    tb.cnt = tbl + (kMaxExperts + 2);
    tb.off = tbl + 2 * (kMaxExperts + 2);
    tb.base = tbl + 3 * (kMaxExperts + 2);
    tb.hdr = tbl + 4 * (kMaxExperts + 2);
    volatile int *abort_flag = tb.hdr + 2;
    uint64_t *bars = reinterpret_cast<uint64_t *>(tb.hdr + 16);
    uint64_t *full = bars, *empty = bars + kStages, *table_ready = bars + 2 * kStages;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    // Only the gate/up kernel runs shared-expert items before the slot table exists (they
    // need no routing).  The down kernel builds its table at once (no wait involved) and
    // its fused combine reads the table, so every one of its items goes through it.
    const int n_sh_items = GU ? shared_items<GU>(p) : 0;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init(table_ready, 1);
        *abort_flag = 0;
        tb.hdr[3] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ======================================================== producer warp
        const CUtensorMap *mA0 = GU ? &maps.g : &maps.d;
        const CUtensorMap *mA1 = &maps.u;
        const CUtensorMap *mS0 = GU ? &maps.sh_g : &maps.sh_d;
        const CUtensorMap *mS1 = &maps.sh_u;
        const CUtensorMap *bA0 = GU ? &maps.gb : &maps.db;
        const CUtensorMap *bA1 = &maps.ub;
        const CUtensorMap *bS0 = GU ? &maps.sh_gb : &maps.sh_db;
        const CUtensorMap *bS1 = &maps.sh_ub;
        const uint64_t pol = l2_evict_first_policy();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, have_table = false;
        int total = n_sh_items;
        int issued_phase[kStages];
        bool unconfirmed[kStages];
        for (int s = 0; s < kStages; ++s) unconfirmed[s] = false, issued_phase[s] = 0;
        for (int i = blockIdx.x; ok; i += G) {
            if (i >= n_sh_items && !have_table) {
                if (GU) pdl_wait();
                build_slot_table<GU>(p, tb);
                if (lane == 0) mbar_arrive(table_ready);
                have_table = true;
                total = tb.hdr[1];
                if (GU) pdl_trigger();
            }
            if (i >= total) break;
            if (lane == 0) {
                const Item it = (i < n_sh_items) ? shared_item<GU>(p, i) : decode_item<GU>(p, tb, i);
                const bool sh = it.e < 0;
                const int ez = sh ? 0 : it.e;
                const int Kb = it.K / 2;
                const int nst = (Kb + kStageK - 1) / kStageK;
                for (int s = 0; s < nst; ++s) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) { ok = false; break; }
                    unconfirmed[stage] = false;
                    const int kb0 = s * kStageK;
                    const int nbox = min(kBoxesPerStage, (Kb - kb0 + kBoxBytes - 1) / kBoxBytes);
                    uint32_t tx = C::kMats * nbox * kBoxSmem + (C::kNv ? C::kMats * kScaleBoxSmem : 0);
                    mbar_arrive_expect_tx(&full[stage], tx);
                    unsigned char *st = ring + (size_t)stage * C::kStageBytes;
#pragma unroll
                    for (int m = 0; m < C::kMats; ++m) {
                        const CUtensorMap *map = sh ? (m ? mS1 : mS0) : (m ? mA1 : mA0);
                        for (int b = 0; b < nbox; ++b)
                            tma_load_3d(st + (m * kBoxesPerStage + b) * kBoxSmem, map, &full[stage],
                                        kb0 + b * kBoxBytes, it.row0, ez, pol);
                        if (C::kNv) {
                            const CUtensorMap *bm = sh ? (m ? bS1 : bS0) : (m ? bA1 : bA0);
                            tma_load_3d(st + C::kCodeBytes + m * 1024, bm, &full[stage],
                                        s * kScaleRowBytes, it.row0, ez, pol);
                        }
                    }
                    issued_phase[stage] = phase;
                    unconfirmed[stage] = true;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) *abort_flag = 1;
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (*abort_flag) ok = false;
        }
        if (!have_table && lane == 0) mbar_arrive(table_ready);  // nothing left: release consumers
        if (lane == 0 && !ok) {
            // let copies still in flight land before the CTA may exit
            for (int s = 0; s < kStages; ++s)
                if (unconfirmed[s]) mbar_wait(&full[s], issued_phase[s], p.status, 10000000ull);
        }
        return;
    }

    // ============================================================ consumer warps
    const int g = lane >> 2, tq = lane & 3;
    const int ctid = tid;   // 0..127
    int stage = 0;
    uint32_t phase = 0;
    bool have_table = false;
    int total = n_sh_items;
    // ldmatrix lane address pieces
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int lch = lane >> 4;
    const int box = warp >> 1;
    const int cbase = (warp & 1) * 4;

    // cfail is written only by consumer warps and read only after a consumer barrier,
    // so all four warps take the same exit decision and meet at the same barriers.
    volatile int *cfail = tb.hdr + 3;
    for (int i = blockIdx.x;; i += G) {
        if (i >= n_sh_items && !have_table) {
            if (!mbar_wait(table_ready, 0, p.status)) {
                *cfail = 1;
                *abort_flag = 1;
            }
            consumer_sync();
            if (*cfail) break;
            have_table = true;
            total = tb.hdr[1];
            if (GU) {
                pdl_wait();     // h, topk and the routed buckets come from the router
                pdl_trigger();
            }
        }
        if (i >= total) break;
        const Item it = (i < n_sh_items) ? shared_item<GU>(p, i) : decode_item<GU>(p, tb, i);
        const bool sh = it.e < 0;
        const int Kb = it.K / 2;
        const int nst = (Kb + kStageK - 1) / kStageK;
        const int nN = (it.ntok + 7) >> 3;

        // B-operand rows of this thread's tokens (one per n-tile: column 8n + g)
        const uint16_t *brow[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int col = 8 * n + g;
            brow[n] = nullptr;
            if (col < it.ntok) {
                const int bpos = it.tok0 + col;
                if (GU) {
                    int t = bpos;
                    if (!sh) {
                        const int a = __ldg(p.perm + it.boff + bpos);
                        t = (a >= 0 && a < p.T * p.k) ? a / p.k : -1;
                        if (t < 0) record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                    }
                    if (t >= 0) brow[n] = p.x + (size_t)t * p.H;
                } else {
                    brow[n] = sh ? reinterpret_cast<const uint16_t *>(p.h_sh) + (size_t)bpos * p.I_sh
                                 : reinterpret_cast<const uint16_t *>(p.h) + (size_t)(it.boff + bpos) * p.I;
                }
            }
        }
        if (!GU && i == blockIdx.x) pdl_wait();   // h is produced by the gate/up kernel

        float acc[C::kMats][4][4];
#pragma unroll
        for (int m = 0; m < C::kMats; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[m][n][c] = 0.f;

        bool ok = true;
        for (int s = 0; s < nst; ++s) {
            if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
            const unsigned char *st = ring + (size_t)stage * C::kStageBytes;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int cc = cbase + 2 * q;                       // chunk pair (cc, cc+1)
                const int kbyte = s * kStageK + box * kBoxBytes + cc * 16;
                if (kbyte >= Kb) continue;
                const int ch = cc + lch;
                const uint32_t off = lrow * kBoxBytes + (((ch ^ (lrow & 7)) & 7) << 4);
                uint32_t A[C::kMats][2][2][4];   // [mat][chunk][row g / g+8][pairs]
#pragma unroll
                for (int m = 0; m < C::kMats; ++m) {
                    uint32_t r0, r1, r2, r3;
                    ldmatrix_x4(r0, r1, r2, r3,
                                smem_u32(st + (m * kBoxesPerStage + box) * kBoxSmem) + off);
                    if (C::kNv) {
                        const unsigned char *sc = st + C::kCodeBytes + m * 1024;
                        const int cis = box * 8 + cc;                 // chunk index in stage
                        const int b0 = 2 * cis + (tq >> 1);
                        const uint32_t s00 = e4m3_to_half2(sc[g * kScaleRowBytes + b0]);
                        const uint32_t s10 = e4m3_to_half2(sc[(g + 8) * kScaleRowBytes + b0]);
                        const uint32_t s01 = e4m3_to_half2(sc[g * kScaleRowBytes + b0 + 2]);
                        const uint32_t s11 = e4m3_to_half2(sc[(g + 8) * kScaleRowBytes + b0 + 2]);
                        dequant_nvfp4_word(r0, s00, A[m][0][0]);
                        dequant_nvfp4_word(r1, s10, A[m][0][1]);
                        dequant_nvfp4_word(r2, s01, A[m][1][0]);
                        dequant_nvfp4_word(r3, s11, A[m][1][1]);
                    } else {
                        dequant_int4_word(r0, A[m][0][0]);
                        dequant_int4_word(r1, A[m][0][1]);
                        dequant_int4_word(r2, A[m][1][0]);
                        dequant_int4_word(r3, A[m][1][1]);
                    }
                }
                const int kel = 2 * kbyte;   // first weight index of chunk cc
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    if (n >= nN) break;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint4 X = make_uint4(0, 0, 0, 0);
                        if (brow[n]) X = __ldg(reinterpret_cast<const uint4 *>(brow[n] + kel + 32 * c + 8 * tq));
                        uint32_t b00, b01, b10, b11;
                        if (GU && FMT == MOE_FMT_INT4_ROWSCALE) {
                            b00 = pack_lo(X.x, X.z);
                            b01 = pack_hi(X.x, X.z);
                            b10 = pack_lo(X.y, X.w);
                            b11 = pack_hi(X.y, X.w);
                        } else {
                            b00 = X.x;
                            b01 = X.y;
                            b10 = X.z;
                            b11 = X.w;
                        }
#pragma unroll
                        for (int m = 0; m < C::kMats; ++m) {
                            mma_16816(acc[m][n], A[m][c][0][0], A[m][c][1][0], A[m][c][0][1],
                                      A[m][c][1][1], b00, b01);
                            mma_16816(acc[m][n], A[m][c][0][2], A[m][c][1][2], A[m][c][0][3],
                                      A[m][c][1][3], b10, b11);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) {
            *cfail = 1;
            *abort_flag = 1;
        }

        // ---------------------------------------------------------------- epilogue
        // partial sums of the four K-slices -> shared memory [warp][mat][col][row]
#pragma unroll
        for (int m = 0; m < C::kMats; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                if (n >= nN) break;
                float *r = red + ((warp * C::kMats + m) * kTokChunk) * kRowTile;
                const int c0 = 8 * n + 2 * tq;
                r[c0 * kRowTile + g] = acc[m][n][0];
                r[(c0 + 1) * kRowTile + g] = acc[m][n][1];
                r[c0 * kRowTile + g + 8] = acc[m][n][2];
                r[(c0 + 1) * kRowTile + g + 8] = acc[m][n][3];
            }
        consumer_sync();
        if (*cfail) break;
        for (int o = ctid; o < it.ntok * kRowTile; o += kConsumerWarps * 32) {
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
                float sg, su;
                if (FMT == MOE_FMT_NVFP4) {
                    sg = sh ? p.wt.sh_g_scale[0] : p.wt.g_scale[it.e];
                    su = sh ? p.wt.sh_u_scale[0] : p.wt.u_scale[it.e];
                } else {
                    sg = sh ? p.wt.sh_g_scale[row] : p.wt.g_scale[(size_t)it.e * p.I + row];
                    su = sh ? p.wt.sh_u_scale[row] : p.wt.u_scale[(size_t)it.e * p.I + row];
                }
                const float gv = v0 * sg, uv = v1 * su;
                const float hv = gv / (1.f + expf(-gv)) * uv;
                __half *dst = sh ? p.h_sh + (size_t)bpos * p.I_sh : p.h + (size_t)(it.boff + bpos) * p.I;
                dst[h_pos<FMT>(row)] = __float2half_rn(hv);
            } else {
                float sd;
                if (FMT == MOE_FMT_NVFP4) sd = sh ? p.wt.sh_d_scale[0] : p.wt.d_scale[it.e];
                else sd = sh ? p.wt.sh_d_scale[row] : p.wt.d_scale[(size_t)it.e * p.H + row];
                const float yv = v0 * sd;
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

        if (!GU && p.fuse_combine) {
            // the last item to finish a 16-row tile combines it: y = shared + sum_j w_j y_j
            __shared__ int s_last;
            const int tile = it.row0 / kRowTile;
            if (ctid == 0) {
                int target = 0;   // items that write this row tile: every token chunk of every slot
                for (int s2 = 0; s2 < tb.hdr[0]; ++s2) target += (tb.cnt[s2] + kTokChunk - 1) / kTokChunk;
                __threadfence();
                const unsigned old = atomicInc(p.row_counters + tile, (unsigned)target - 1u);
                s_last = (old == (unsigned)target - 1u);
            }
            consumer_sync();
            if (s_last) {
                __threadfence();
                for (int o = ctid; o < p.T * kRowTile; o += kConsumerWarps * 32) {
                    const int t = o / kRowTile, row = it.row0 + o % kRowTile;
                    float yv = p.n_shared ? __ldcg(p.y_shared + (size_t)t * p.H + row) : 0.f;
                    for (int j = 0; j < p.k; ++j)
                        yv = fmaf(__ldg(p.topk_w + (size_t)t * p.k + j),
                                  __ldcg(p.y_assign + ((size_t)t * p.k + j) * p.H + row), yv);
                    p.y[(size_t)t * p.H + row] = __half_as_ushort(__float2half_rn(yv));
                }
            }
            consumer_sync();
        }
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
template <int FMT, bool GU>
static cudaError_t launch_ffn_t(const LayerMaps &maps, const FfnParams &p, int grid, bool pdl,
                                cudaStream_t s)
{
    using C = FfnCfg<FMT, GU>;
    auto kern = ffn_kernel<FMT, GU>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kFfnThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, maps, p);
}

size_t ffn_smem_bytes(int fmt, bool gu)
{
    if (fmt == MOE_FMT_NVFP4) return gu ? FfnCfg<1, true>::kSmem : FfnCfg<1, false>::kSmem;
    return gu ? FfnCfg<0, true>::kSmem : FfnCfg<0, false>::kSmem;
}

cudaError_t ffn_occupancy(int fmt, bool gu, int *blocks_per_sm)
{
    const size_t smem = ffn_smem_bytes(fmt, gu);
    cudaError_t e;
    if (fmt == MOE_FMT_NVFP4) {
        if (gu) {
            cudaFuncSetAttribute(ffn_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, ffn_kernel<1, true>, kFfnThreads, smem);
        } else {
            cudaFuncSetAttribute(ffn_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, ffn_kernel<1, false>, kFfnThreads, smem);
        }
    } else {
        if (gu) {
            cudaFuncSetAttribute(ffn_kernel<0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, ffn_kernel<0, true>, kFfnThreads, smem);
        } else {
            cudaFuncSetAttribute(ffn_kernel<0, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, ffn_kernel<0, false>, kFfnThreads, smem);
        }
    }
    return e;
}

cudaError_t launch_ffn(const LayerMaps &maps, const FfnParams &p, bool gate_up, int grid, bool pdl,
                       cudaStream_t s)
{
    if (p.fmt == MOE_FMT_NVFP4)
        return gate_up ? launch_ffn_t<1, true>(maps, p, grid, pdl, s)
                       : launch_ffn_t<1, false>(maps, p, grid, pdl, s);
    return gate_up ? launch_ffn_t<0, true>(maps, p, grid, pdl, s)
                   : launch_ffn_t<0, false>(maps, p, grid, pdl, s);
}

cudaError_t launch_wait_timeout(int *status, unsigned long long max_iters, cudaStream_t s)
{
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, max_iters);
    return cudaGetLastError();
}

}  // namespace moe
