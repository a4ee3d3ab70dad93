// moe_expert.cuh -- pieces of the expert kernels shared by the per-step kernels
// (moe_ffn.cu) and the fused decode-layer kernel (moe_fused.cu): ring geometry, the
// int4 / NVFP4 chunk-pair inner loops on the warp MMAs, the consumer barrier and the
// conversion of finished h rows to int8 limbs.
#pragma once

#include <cuda_fp16.h>
#include <math.h>

#include "moe_device.cuh"
#include "moe_internal.h"

#ifndef MOE_CHAINS
#define MOE_CHAINS 1
#endif
#ifndef MOE_MIN_CTAS
#define MOE_MIN_CTAS 2
#endif

namespace moe {

constexpr int kConsumerWarps = 4;
constexpr int kFfnThreads = (kConsumerWarps + 1) * 32;
constexpr int kBoxBytes = 128;          // K bytes per TMA box = swizzle span
constexpr int kBoxSmem = kRowTile * kBoxBytes;     // 2 KB
constexpr int kScaleBoxBytes = kBoxBytes / 8;      // NVFP4: one E4M3 per 16 weights = 16 B
constexpr int kScaleBoxSmem = kRowTile * kScaleBoxBytes;   // 256 B
constexpr int kMatStage = kConsumerWarps * kBoxSmem;       // 8 KB of codes per matrix

template <int FMT, bool GU, int KS, int NNMAX>
struct FfnCfg {
    static constexpr int kMats = GU ? 2 : 1;
    static constexpr int kRW = kConsumerWarps / KS;
    static constexpr bool kNv = FMT == MOE_FMT_NVFP4;
    // decode variant of the row-scaled formats: the int8 tensor path (weights as s8 bytes,
    // activations as three int8 limbs; items of at most 8 tokens, KS = 1).  int8 and int2
    // weights run only this variant.
    static constexpr bool kLimbs = row_scaled(FMT) && NNMAX == 1 && KS == 1;
    // K boxes (128 bytes wide) per matrix and stage: a stage covers whole 256-value limb
    // blocks -- int8 two boxes (256 values), int4 two (512), int2 one (512).  Fewer, larger
    // stages cost less per byte (one full/empty handshake, one B copy per token and stage):
    // measured on B200, 16-KB down stages beat 8-KB ones by 8% (decode8), and 32 KB is worse
    // again (fewer stages in flight per CTA).
    static constexpr int kBoxesK = !kLimbs ? 1 : FMT == MOE_FMT_INT2_ROWSCALE ? 1 : 2;
    static constexpr int kMatBytes = kBoxesK * kMatStage;     // one matrix's codes per stage
    static constexpr int kStageK = KS * kBoxesK * kBoxBytes;  // K bytes per stage
    static constexpr int kStageVals = kStageK * 8 / code_bits(FMT);   // K values per stage
    static constexpr int kGroups = kStageVals / 64;           // 64-value groups per stage
    static constexpr int kCodeShift = FMT == MOE_FMT_INT8_ROWSCALE ? 0 : FMT == MOE_FMT_INT2_ROWSCALE ? 6 : 4;
    static constexpr int kCodeBytes = kMats * kMatBytes;
    static constexpr int kScaleBytes = kNv ? kMats * kConsumerWarps * kScaleBoxSmem : 0;
    // decode variant: the producer also copies each stage's slice of the (up to 8) token
    // rows of the B operand into shared memory, one row per token: fp16 values padded to
    // 16 bytes, or the limb blocks of the stage's K values (768 bytes per 256 values)
    static constexpr bool kSmemB = NNMAX == 1 && KS == 1;
    static constexpr int kBRow = kLimbs ? kStageVals / kLimbBlockK * kLimbBlockBytes : 4 * kStageK + 16;
    static constexpr int kBBytes = kSmemB ? 8 * kBRow : 0;      // per stage, after the ring (at most)
    static constexpr int kStageBytes = ((kCodeBytes + kScaleBytes) + 1023) / 1024 * 1024;
    // Ring depth.  Weights in flight per SM decide the bandwidth (DRAM latency under full
    // load is about 2.5 us); the int8 path sizes its ring at launch (up to kStagesMax
    // stages, as many as fit beside a second CTA on the SM, given the B rows per stage).
    static constexpr int kStages = GU ? (kSmemB ? 3 : 4) : 5;
    static constexpr int kStagesCap = kLimbs ? ((GU ? 6 : 12) / kBoxesK < 2 ? 2 : (GU ? 6 : 12) / kBoxesK) : kStages;
    static constexpr int kZeroRow = kSmemB ? kBRow : 0;   // zero row read by padding lanes
    static constexpr int kRedFloats = KS > 1 ? kConsumerWarps * kMats * kTokChunk * kRowTile : 0;
};

// Resident CTAs per SM an expert kernel is compiled for.  The int8-path down kernels run
// three (about 73 KB of ring each): their consumers, not the weight stream, pace them --
// measured on B200 with the same bytes in flight per SM, one CTA per SM instead of two
// made the down kernel 25-48% slower (decode1, decode8), and three instead of two made
// it 3-11% faster.  The others run two.
template <int FMT, bool GU, int KS, int NNMAX>
__host__ __device__ constexpr int ffn_min_ctas()
{
    return (!GU && FfnCfg<FMT, GU, KS, NNMAX>::kLimbs) ? 3 : MOE_MIN_CTAS;
}

constexpr int kStagesMax = 16;   // ring stages any launch may use (mbarrier slots)
constexpr int kItemQ = 4;        // work items the producer may announce ahead of the consumers
constexpr int kMaxConvRows = 64; // h rows one conversion handles (tokens of a work item)

// dynamic shared memory of one CTA: ring (weights, then B rows) + zero row + reduction +
// slot table + header/barriers
template <int FMT, bool GU, int KS, int NNMAX>
__host__ __device__ constexpr size_t ffn_smem(int E, int stages, int b_stage)
{
    using C = FfnCfg<FMT, GU, KS, NNMAX>;
    return 1024 + (size_t)stages * (C::kStageBytes + b_stage) + C::kZeroRow + (size_t)C::kRedFloats * 4 +
           (size_t)4 * 4 * (E + 2) + 64 + 8 + (2 * kStagesMax + 1 + 2 * kItemQ) * 8;
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

// named barrier of the four consumer warps (the producer warp never joins it); NT: the
// threads that meet there (the tensor-memory kernel's converter warps use it too)
template <int NT = kConsumerWarps * 32, int ID = 1>
__device__ __forceinline__ void consumer_sync()
{
    asm volatile("bar.sync %0, %1;" ::"n"(ID), "r"(NT) : "memory");
}

// row-scaled formats: the fp32 scale of row `row`; NVFP4: the fp32 scale of the whole matrix
template <int FMT>
__device__ __forceinline__ float mat_scale(const float *scales, int e, int rows, int row)
{
    const int ez = e < 0 ? 0 : e;
    if (FMT == MOE_FMT_NVFP4) return scales[ez];
    return scales[(size_t)ez * rows + row];
}

// Per-thread constants of a consumer warp.
struct Lane {
    int lane, g, tq, warp, rw, ks, bx;
    uint32_t off[4];   // swizzled ldmatrix offsets of chunk pairs 0..3 inside a box
    DequantK dk;
};

// B-operand row of each of a thread's four n-tiles
struct BRows {
    const uint16_t *r[4];
};

// One chunk pair (64 weights of each of the warp's 16 rows and of each matrix): ldmatrix,
// dequantise in registers, NN n-tiles of mma.  X0/X1 hold the n-tile-0 B fragments.
// independent accumulator chains per (matrix, n-tile): mma.sync results feed the next
// mma on the same accumulator, so one chain per matrix would serialise a stage's 16 mma
template <int NN>
struct Chains {
    static constexpr int P = MOE_CHAINS;
};

template <int FMT, bool GU, int KS, int NN, bool PERM>
__device__ __forceinline__ void chunk_pair(const unsigned char *st, uint32_t abase, const Lane &L, int q, int kel,
                                           const uint4 &X0, const uint4 &X1, const BRows &brow,
                                           float (&acc)[GU ? 2 : 1][NN][Chains<NN>::P][4])
{
    using C = FfnCfg<FMT, GU, KS, 1>;   // the values used here do not depend on NNMAX
    uint32_t A[C::kMats][2][2][4];   // [mat][chunk][row g / g+8][pairs]
#pragma unroll
    for (int m = 0; m < C::kMats; ++m) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(r0, r1, r2, r3, abase + m * kMatStage + L.off[q]);
        if constexpr (C::kNv) {
            const unsigned char *sc = st + C::kCodeBytes + (m * kConsumerWarps + L.bx) * kScaleBoxSmem;
            const int b0 = 4 * q + (L.tq >> 1);       // block of (chunk 2q, word tq)
            const uint32_t s00 = e4m3_to_half2(sc[L.g * kScaleBoxBytes + b0]);
            const uint32_t s10 = e4m3_to_half2(sc[(L.g + 8) * kScaleBoxBytes + b0]);
            const uint32_t s01 = e4m3_to_half2(sc[L.g * kScaleBoxBytes + b0 + 2]);
            const uint32_t s11 = e4m3_to_half2(sc[(L.g + 8) * kScaleBoxBytes + b0 + 2]);
            dequant_nvfp4_word(r0, s00, A[m][0][0]);
            dequant_nvfp4_word(r1, s10, A[m][0][1]);
            dequant_nvfp4_word(r2, s01, A[m][1][0]);
            dequant_nvfp4_word(r3, s11, A[m][1][1]);
        } else {
            dequant_int4_word(r0, A[m][0][0], L.dk);
            dequant_int4_word(r1, A[m][0][1], L.dk);
            dequant_int4_word(r2, A[m][1][0], L.dk);
            dequant_int4_word(r3, A[m][1][1], L.dk);
        }
    }
#pragma unroll
    for (int n = 0; n < NN; ++n) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 X = n == 0 ? (c == 0 ? X0 : X1)
                                   : __ldg(reinterpret_cast<const uint4 *>(brow.r[n] + kel + 32 * c + 8 * L.tq));
            uint32_t b00, b01, b10, b11;
            if constexpr (PERM) {
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
            constexpr int P = Chains<NN>::P;
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
                mma_16816(acc[m][n][(2 * c) % P], A[m][c][0][0], A[m][c][1][0], A[m][c][0][1], A[m][c][1][1], b00, b01);
                mma_16816(acc[m][n][(2 * c + 1) % P], A[m][c][0][2], A[m][c][1][2], A[m][c][0][3], A[m][c][1][3], b10, b11);
            }
        }
    }
}

// int8 path, the A operand of one 64-value group q of a stage, for one matrix whose
// stage codes start at shared address `mbase` (the warp's 16-row box of each K box):
// ev[i] / od[i] hold, as s8 bytes 2^shift x code, the even / odd elements of the 8 K
// values 64 q + 32 c + 8 tq .. +7 of row g (i = 2c) or g + 8 (i = 2c + 1) -- the order of
// the limb bytes of the B operand.
//  int4: ldmatrix words (chunk 2q + c of rows g, g + 8), nibbles moved to the top of bytes;
//  int8: the 8 bytes of each (row, c), split into even and odd bytes;
//  int2: the 16 bits of each (row, c); rows g and g + 8 are joined in one word and each
//        2-bit code is moved to the top two bits of its byte.
// Rows are 128 bytes with the 128-byte swizzle (16-byte unit u of row r at u ^ (r % 8)).
template <int FMT>
__device__ __forceinline__ void limb_a_words(uint32_t mbase, const Lane &L, int q, uint32_t (&ev)[4],
                                             uint32_t (&od)[4])
{
    if constexpr (FMT == MOE_FMT_INT8_ROWSCALE) {
        const uint32_t base = mbase + (q >> 1) * kMatStage;   // K box of the group
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = L.g + 8 * (i & 1), c = i >> 1;
            const int u = 4 * (q & 1) + 2 * c + (L.tq >> 1);
            uint32_t lo, hi;
            asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                         : "=r"(lo), "=r"(hi)
                         : "r"(base + r * kBoxBytes + ((u ^ (r & 7)) << 4) + 8 * (L.tq & 1)));
            ev[i] = __byte_perm(lo, hi, 0x6420);
            od[i] = __byte_perm(lo, hi, 0x7531);
        }
    } else if constexpr (FMT == MOE_FMT_INT2_ROWSCALE) {
        constexpr uint32_t kTop = 0xC0C0C0C0u;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t v[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = L.g + 8 * h;
                unsigned short b;
                asm volatile("ld.shared.u16 %0, [%1];"
                             : "=h"(b)
                             : "r"(mbase + r * kBoxBytes + ((q ^ (r & 7)) << 4) + 8 * c + 2 * L.tq));
                v[h] = b;
            }
            // bytes 0, 1: row g (codes 0..3, 4..7); bytes 2, 3: row g + 8
            const uint32_t w = __byte_perm(v[0], v[1], 0x5410);
            // top two bits of byte b after the shift: code 0 / 4 (<< 6), 2 / 6 (<< 2),
            // 1 / 5 (<< 4), 3 / 7 (no shift) of the 16-bit row in bytes 2b', 2b' + 1
            const uint32_t s6 = w << 6, s2 = w << 2, s4 = w << 4;
            ev[2 * c] = __byte_perm(s6, s2, 0x5140) & kTop;
            ev[2 * c + 1] = __byte_perm(s6, s2, 0x7362) & kTop;
            od[2 * c] = __byte_perm(s4, w, 0x5140) & kTop;
            od[2 * c + 1] = __byte_perm(s4, w, 0x7362) & kTop;
        }
    } else {
        uint32_t r[4];
        ldmatrix_x4(r[0], r[1], r[2], r[3], mbase + (q >> 2) * kMatStage + L.off[q & 3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) int4_word_to_s8x16(r[i], ev[i], od[i]);
    }
}

// int8 path, one 64-value group q of a stage: 64 K values of each of the warp's 16 rows
// and of each matrix.  The A words (limb_a_words) are s8 bytes 2^shift x code: even
// elements feed one mma, odd elements a second one, with the matching limb bytes of the
// B operand (the 16 bytes at 64 (q % 4) of the group's limb block: even elements of the
// two 32-value halves, then odd ones).  NN = 1: one n-tile whose columns are
// (limb, token) = (g / 2, g % 2); NN = 3: n-tile = limb, column = token.  The two mma
// accumulate 2^shift x sum(code * limb) exactly in s32, in two independent chains (even
// and odd elements) so that a stage's mma do not serialise.
template <int FMT, bool GU, int NN>
__device__ __forceinline__ void chunk_pair_limbs(uint32_t abase, const Lane &L, int q, const uint4 (&Bq)[NN],
                                                 int (&acc)[2][GU ? 2 : 1][NN][4])
{
    using C = FfnCfg<FMT, GU, 1, 1>;
    constexpr int M = GU ? 2 : 1;
    uint32_t ev[M][4], od[M][4];
#pragma unroll
    for (int m = 0; m < M; ++m) limb_a_words<FMT>(abase + m * C::kMatBytes, L, q, ev[m], od[m]);
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

// int8 path, gate/up: the ntok h rows of a finished token chunk (fp16, natural order,
// K values each) -> int8 limb rows and their scales.  The rows' largest magnitudes were
// gathered by the items that wrote them (atomicMax on the float bits, reset here for the
// next call).  The four consumer warps.
template <int NT, int BAR = 1>
__device__ __noinline__ void convert_h_rows(const __half *src0, size_t src_stride, unsigned char *dst0, float *scale0,
                                            unsigned *amax0, int ntok, int K, int ltid)
{
    __shared__ float s_m[kMaxConvRows];
    if (ltid < ntok) {
        s_m[ltid] = __uint_as_float(__ldcg(amax0 + ltid));
        amax0[ltid] = 0u;
    }
    consumer_sync<NT, BAR>();
    const int nb = (K + kLimbBlockK - 1) / kLimbBlockK;
    const size_t row_bytes = (size_t)nb * kLimbBlockBytes;
    for (int j = 0; j < ntok; ++j) {
        const int sh = limb_shift(s_m[j]);
        const float scale = pow2f(sh);
        const __half *src = src0 + j * src_stride;
        unsigned char *dst = dst0 + j * row_bytes;
        for (int k8 = 8 * ltid; k8 < nb * kLimbBlockK; k8 += 8 * NT) {
            const uint4 v = k8 < K ? __ldcg(reinterpret_cast<const uint4 *>(src + k8)) : make_uint4(0u, 0u, 0u, 0u);
            limb_encode8(v, scale, dst + (size_t)(k8 / kLimbBlockK) * kLimbBlockBytes, k8 % kLimbBlockK);
        }
        if (ltid == 0) scale0[j] = pow2f(-sh);
    }
    consumer_sync<NT, BAR>();   // s_m is reused by the next conversion
}

}  // namespace moe
