// moe_device.cuh -- device-side building blocks shared by the MoE kernels (sm_100a).
//
// mbarrier waits are bounded (iteration count and %globaltimer deadline); a wait that
// gives up records MOE_ERR_DEVICE_TIMEOUT in the layer's status word and lets the
// kernel return instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// ------------------------------------------------------------------ limits & status
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s: never reached when healthy
constexpr unsigned long long kWaitMaxIters = 1ull << 30;

__device__ __forceinline__ void record_error(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000000;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false (after recording
// MOE_ERR_DEVICE_TIMEOUT) if the barrier did not complete in time.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *status,
                                          unsigned long long timeout_ns = kWaitTimeoutNs,
                                          unsigned long long max_iters = kWaitMaxIters)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (unsigned long long it = 1; it < max_iters; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0 && globaltimer_ns() - t0 > timeout_ns) break;
    }
    record_error(status, MOE_ERR_DEVICE_TIMEOUT);
    return false;
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 3-D tiled bulk tensor copy global -> shared, completing on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
        "l"(policy)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ PDL
// Programmatic dependent launch: wait for the prerequisite grid (no-op without one)
// and allow dependents to be scheduled.
// Increment of a completion counter with acquire-release semantics at GPU scope (wraps
// to 0 after `last`, as atomicInc); returns the old value.  Writers publish what they
// (and, through a preceding barrier, their block) stored; the last arriver sees it all.
__device__ __forceinline__ unsigned atom_inc_acq_rel(unsigned *ctr, unsigned last)
{
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;" : "=r"(old) : "l"(ctr), "r"(last) : "memory");
    return old;
}

// 1-D bulk copy global -> shared completing on an mbarrier (16-byte aligned, size % 16 == 0)
__device__ __forceinline__ void bulk_copy(void *smem_dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// 16-byte asynchronous copy global -> shared through L2 only (Ampere-style, per thread),
// with commit groups and a wait for all but the newest N groups
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// the same with a run-time count (0 .. 7)
__device__ __forceinline__ void cp_async_wait_n(int n)
{
    switch (n) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    case 6: cp_async_wait<6>(); break;
    default: cp_async_wait<7>(); break;
    }
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;"); }

// ------------------------------------------------------------------ warp MMA
__device__ __forceinline__ void ldmatrix_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                            uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D = A(16x16, f16, row) * B(16x8, f16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ dequantisation
// Constants of the int4 dequantisation.  They are passed to the kernels at run time so
// that each lives in one register (or a constant-bank operand) for the whole kernel: as
// compile-time literals the compiler splits the fused logic ops and rematerialises the
// literals, which doubles the instruction count of the inner loop.
struct DequantK {
    uint32_t m_lo;    // 0x000F000F: low nibble of bytes 0 and 2
    uint32_t m_hi;    // 0x00F000F0: high nibble of bytes 0 and 2
    uint32_t x_lo;    // 0x64086408: 0x6400 (fp16 1024) | bit 3 of the low nibble
    uint32_t x_hi;    // 0x64806480: 0x6400 | bit 3 of the high nibble
    uint32_t h1032;   // fp16x2 1032
    uint32_t h1_16;   // fp16x2 1/16
    uint32_t hm72;    // fp16x2 -72
};

// int4 (two's complement, 8 codes in a 32-bit word, element i in bits 4i..4i+3) to four
// fp16 pairs, exactly.  Each code q is placed in the mantissa of the fp16 number 1024
// (exponent trick: 0x6400 | m == 1024 + m) as q + 8: flipping bit 3 of a two's complement
// nibble gives q + 8, and since the flip bit lies under the mask and 0x6400 outside it,
// (w & mask) ^ (0x6400 | flip) is a single 3-input logic op.  The bias is then removed
// with one fp16 subtract (low nibbles) or one fma with 1/16 (high nibbles, which sit
// 4 bits higher).  Five integer and four fp16 ops per 8 weights.  Output pairs hold
// elements (0,4), (1,5), (2,6), (3,7) of the word: callers order the other operand alike.
__device__ __forceinline__ void dequant_int4_word(uint32_t w, uint32_t (&r)[4], const DequantK &k)
{
    const uint32_t hi = w >> 8;
    uint32_t t0, t1, t2, t3;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t0) : "r"(w), "r"(k.m_lo), "r"(k.x_lo));   // (a & b) ^ c
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t1) : "r"(w), "r"(k.m_hi), "r"(k.x_hi));
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t2) : "r"(hi), "r"(k.m_lo), "r"(k.x_lo));
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t3) : "r"(hi), "r"(k.m_hi), "r"(k.x_hi));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r[0]) : "r"(t0), "r"(k.h1032));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r[1]) : "r"(t1), "r"(k.h1_16), "r"(k.hm72));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r[2]) : "r"(t2), "r"(k.h1032));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r[3]) : "r"(t3), "r"(k.h1_16), "r"(k.hm72));
}

// NVFP4 word (8 E2M1 codes) times one E4M3 block scale (given as an fp16 pair) to four
// fp16 pairs, exactly (an E2M1 value times an E4M3 value has at most 6 significant bits
// and lies in [2^-10, 2688]).  Output pairs hold elements (0,1), (2,3), (4,5), (6,7).
__device__ __forceinline__ void dequant_nvfp4_word(uint32_t w, uint32_t scale2, uint32_t (&r)[4])
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
        : "r"(w));
#pragma unroll
    for (int i = 0; i < 4; ++i) asm("mul.rn.f16x2 %0, %0, %1;" : "+r"(r[i]) : "r"(scale2));
}

// one E4M3 byte -> the fp16 pair (v, v)
__device__ __forceinline__ uint32_t e4m3_to_half2(uint32_t byte)
{
    uint32_t r;
    const uint16_t two = static_cast<uint16_t>(byte | (byte << 8));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(two));
    return r;
}

// ------------------------------------------------------------------ int8 tensor path
// mma m16n8k32, s8 x s8 -> s32, accumulating in place
__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// An int4 word (8 two's complement codes, element i in bits 4i..4i+3) as two words of
// four s8 bytes each holding 16 x code: the odd elements are already in place in the
// high half of each byte (a byte 0xq0 read as s8 is 16 q), the even ones move there with
// a 4-bit left shift.  Byte j of `even` is element 2j, byte j of `odd` element 2j + 1.
__device__ __forceinline__ void int4_word_to_s8x16(uint32_t w, uint32_t &even, uint32_t &odd)
{
    odd = w & 0xF0F0F0F0u;
    even = (w << 4) & 0xF0F0F0F0u;
}

// Activation limbs.  A row of fp16 values v_k is written as X_k = round(v_k * 2^sh) with
// one power-of-two exponent sh per row chosen so that max |X_k| lies in [2^21, 2^22), and
// X_k = P0 + 256 P1 + 65536 P2 with s8 digits (|P2| <= 64).  Every v_k whose binary
// exponent is at least 11 below the row maximum's is represented exactly; smaller ones
// are rounded to a multiple of 2^-sh (error <= 2^-22 max |v|).  The limbs of a row are
// stored per block of 256 K values as three 256-byte arrays (P0, P1, P2), each in the
// order in which the int8 kernels load their B fragments: the 8 values starting at K
// offset k8 (a multiple of 8 inside the block) go to the word at
// 64 (k8 / 64) + 16 ((k8 / 8) % 4) + 4 ((k8 / 32) % 2) (even elements, bytes in order)
// and to the word 8 bytes further (odd elements).
constexpr int kLimbBlockK = 256;
constexpr int kLimbBlockBytes = 3 * kLimbBlockK;

__device__ __forceinline__ int limb_word_offset(int k8)
{
    return 64 * (k8 >> 6) + 16 * ((k8 >> 3) & 3) + 4 * ((k8 >> 5) & 1);
}

// exponent sh for a row whose largest magnitude is amax (finite); 0 for an all-zero row
__device__ __forceinline__ int limb_shift(float amax)
{
    if (!(amax > 0.f)) return 0;
    const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);  // amax in [2^(e-127), 2^(e-126))
    return 148 - e;
}

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }   // -126 <= e <= 127

// the three limb digits of round(v * scale) (scale = 2^sh)
__device__ __forceinline__ void limb_digits(float v, float scale, int &p0, int &p1, int &p2)
{
    const int X = __float2int_rn(v * scale);
    p0 = static_cast<int>(static_cast<int8_t>(X & 0xFF));
    const int X1 = (X - p0) / 256;     // exact: X - p0 is a multiple of 256
    p1 = static_cast<int>(static_cast<int8_t>(X1 & 0xFF));
    p2 = (X1 - p1) / 256;
}

// Encodes 8 consecutive fp16 values (k8 .. k8+7 of a block) into the block's limb arrays.
__device__ __forceinline__ void limb_encode8(const uint4 v8, float scale, unsigned char *block, int k8)
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&v8);
    uint32_t ev[3] = {0u, 0u, 0u}, od[3] = {0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        int a0, a1, a2, b0, b1, b2;
        limb_digits(f.x, scale, a0, a1, a2);
        limb_digits(f.y, scale, b0, b1, b2);
        ev[0] |= (uint32_t)(a0 & 0xFF) << (8 * j);
        ev[1] |= (uint32_t)(a1 & 0xFF) << (8 * j);
        ev[2] |= (uint32_t)(a2 & 0xFF) << (8 * j);
        od[0] |= (uint32_t)(b0 & 0xFF) << (8 * j);
        od[1] |= (uint32_t)(b1 & 0xFF) << (8 * j);
        od[2] |= (uint32_t)(b2 & 0xFF) << (8 * j);
    }
    const int o = limb_word_offset(k8);
#pragma unroll
    for (int p = 0; p < 3; ++p) {
        *reinterpret_cast<uint32_t *>(block + p * kLimbBlockK + o) = ev[p];
        *reinterpret_cast<uint32_t *>(block + p * kLimbBlockK + o + 8) = od[p];
    }
}

// largest |v| of 8 fp16 values
__device__ __forceinline__ float amax8(const uint4 v8)
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&v8);
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    return m;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// (a.lo16, b.lo16) and (a.hi16, b.hi16)
__device__ __forceinline__ uint32_t pack_lo(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x5410); }
__device__ __forceinline__ uint32_t pack_hi(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7632); }

}  // namespace moe
