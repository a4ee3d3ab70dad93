/*
 * synth.c -- seeded synthetic inputs for the W4A16 quantized-expert MoE layer.
 *
 * This module is shared by the CPU oracle's tests and by the CUDA path's tests and
 * benchmark.  It only draws random numbers and packs them into the storage formats
 * the layer consumes; it contains none of the layer's arithmetic (no dequantisation,
 * no routing, no matmul).
 *
 * Randomness is counter-based: every value is a pure function of
 * (seed, stream, element index), so tensors can be generated in any order, in
 * parallel, and one expert at a time, and the bytes never depend on the thread count.
 * The mixing function is the SplitMix64 output finaliser (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014) applied to
 * key + (index + 1) * golden-gamma.
 *
 * Distributions follow the workload descriptions: fp16 activations ~ N(0,1),
 * router weights ~ N(0, 1/H), selection bias ~ U(lo, hi) or a Zipf(s) ranking,
 * int4 codes uniform on [-8, 7] packed two per byte (low nibble first), fp32 row
 * scales ~ U(0.01, 0.03), and NVFP4 blocks quantised from N(0,1) samples.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t fmix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream)
{
    return fmix64(fmix64(seed + GOLDEN) ^ (stream * 0xD1B54A32D192ED03ULL + 1));
}

static inline uint64_t draw(uint64_t key, uint64_t i)
{
    return fmix64(key + (i + 1) * GOLDEN);
}

/* uniform double in [0, 1) with 53 random bits */
static inline double unit(uint64_t r) { return (double)(r >> 11) * 0x1.0p-53; }

/* standard normal by Box-Muller from draws 2i and 2i+1 of the stream */
static inline double normal_at(uint64_t key, uint64_t i)
{
    double u1 = 1.0 - unit(draw(key, 2 * i));      /* (0, 1] */
    double u2 = unit(draw(key, 2 * i + 1));
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

/* IEEE binary16 encoding with round-to-nearest-even (finite inputs; saturates
 * to +-inf above the largest finite half). */
static uint16_t f64_to_half_rne(double v)
{
    uint16_t sign = 0;
    if (signbit(v)) { sign = 0x8000; v = -v; }
    if (v == 0.0) return sign;
    if (v >= 65520.0) return sign | 0x7C00;
    int e;
    frexp(v, &e);              /* v = f * 2^e, f in [0.5, 1) */
    int ue = e - 1;            /* unbiased exponent of the leading bit */
    if (ue < -14) ue = -14;    /* subnormal range shares the quantum 2^-24 */
    double q = ldexp(1.0, ue - 10);
    double m = nearbyint(v / q);  /* default rounding mode: ties to even */
    /* m in [1024, 2048] for normals, [0, 1024] for subnormals */
    if (m >= 2048.0) { m = 1024.0; ue += 1; }
    if (m < 1024.0) return sign | (uint16_t)m;   /* subnormal (ue == -14) */
    if (ue > 15) return sign | 0x7C00;
    return sign | (uint16_t)(((ue + 15) << 10) | ((int)m - 1024));
}

/* ---------------------------------------------------------------- exports */

void synth_normal_f16(uint64_t seed, uint64_t stream, double std, uint16_t *out, size_t n)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static) if (n > 65536)
    for (size_t i = 0; i < n; i++) out[i] = f64_to_half_rne(std * normal_at(key, i));
}

void synth_normal_f32(uint64_t seed, uint64_t stream, double std, float *out, size_t n)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static) if (n > 65536)
    for (size_t i = 0; i < n; i++) out[i] = (float)(std * normal_at(key, i));
}

void synth_uniform_f32(uint64_t seed, uint64_t stream, double lo, double hi, float *out, size_t n)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static) if (n > 65536)
    for (size_t i = 0; i < n; i++) out[i] = (float)(lo + (hi - lo) * unit(draw(key, i)));
}

/* Uniform random bytes.  Two uniform 4-bit fields per byte make int4 codes that are
 * uniform on [-8, 7] in two's complement, low nibble first. */
void synth_bytes(uint64_t seed, uint64_t stream, uint8_t *out, size_t n)
{
    uint64_t key = stream_key(seed, stream);
    size_t words = n / 8;
#pragma omp parallel for schedule(static) if (words > 8192)
    for (size_t w = 0; w < words; w++) {
        uint64_t r = draw(key, w);
        memcpy(out + 8 * w, &r, 8);
    }
    if (n % 8) {
        uint64_t r = draw(key, words);
        memcpy(out + 8 * words, &r, n % 8);
    }
}

/* Zipf(s) ranking scaled into [lo, hi]: a seeded permutation assigns ranks
 * 1..E to experts; rank r gets z_r = r^-s; the bias is an affine map of z onto
 * [lo, hi] (rank 1 -> hi, rank E -> lo). */
void synth_zipf_bias(uint64_t seed, uint64_t stream, int E, double s, double lo, double hi,
                     float *out)
{
    uint64_t key = stream_key(seed, stream);
    int *perm = (int *)malloc(sizeof(int) * (size_t)E);
    for (int i = 0; i < E; i++) perm[i] = i;
    for (int i = E - 1; i > 0; i--) {          /* Fisher-Yates */
        int j = (int)(draw(key, (uint64_t)i) % (uint64_t)(i + 1));
        int t = perm[i]; perm[i] = perm[j]; perm[j] = t;
    }
    double zmax = 1.0, zmin = pow((double)E, -s);
    for (int r = 1; r <= E; r++) {
        double z = pow((double)r, -s);
        double v = (E > 1) ? lo + (hi - lo) * (z - zmin) / (zmax - zmin) : hi;
        out[perm[r - 1]] = (float)v;
    }
    free(perm);
}

/* Round a positive value onto the FP8 E4M3 (OCP "FN") grid, ties to even,
 * saturating at 448.  Returns the byte; *val receives the rounded value. */
static uint8_t e4m3_encode_pos(double v, double *val)
{
    if (!(v > 0.0)) { *val = 0.0; return 0; }
    int e;
    frexp(v, &e);
    int ue = e - 1;
    if (ue < -6) ue = -6;                 /* subnormals share the quantum 2^-9 */
    double q = ldexp(1.0, ue - 3);
    double m = nearbyint(v / q);          /* 8..16 for normals, 0..8 for subnormals */
    if (m >= 16.0) { m = 8.0; ue += 1; }
    double r = m * ldexp(1.0, ue - 3);
    if (r > 448.0 || ue > 8) { *val = 448.0; return 0x7E; }
    *val = r;
    if (m < 8.0) return (uint8_t)m;       /* subnormal, exponent field 0 */
    return (uint8_t)(((ue + 7) << 3) | ((int)m - 8));
}

/* Round onto the FP4 E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the code with
 * an even mantissa bit, saturating at 6.  Returns the 4-bit code. */
static uint8_t e2m1_encode(double v)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    uint8_t sign = 0;
    if (v < 0) { sign = 8; v = -v; }
    int best = 0;
    double bd = v;
    for (int c = 1; c < 8; c++) {
        double d = fabs(v - mag[c]);
        if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = c; }
    }
    if (best == 0) sign = 0;
    return (uint8_t)(sign | best);
}

/* NVFP4 block quantisation of N(0,1) samples: rows x K values (K a multiple of 16),
 * one E4M3 scale per 16 consecutive K elements of a row, sb = E4M3(amax / 6),
 * codes = E2M1(z / sb), packed two per byte with the low nibble first.
 * codes: rows * K/2 bytes; bscale: rows * K/16 bytes. */
void synth_nvfp4(uint64_t seed, uint64_t stream, int rows, int K, uint8_t *codes,
                 uint8_t *bscale)
{
    uint64_t key = stream_key(seed, stream);
    int nb = K / 16;
#pragma omp parallel for schedule(static) if ((size_t)rows * (size_t)K > 65536)
    for (int r = 0; r < rows; r++) {
        for (int b = 0; b < nb; b++) {
            double z[16], amax = 0.0;
            for (int i = 0; i < 16; i++) {
                z[i] = normal_at(key, (uint64_t)r * (uint64_t)K + (uint64_t)(16 * b + i));
                if (fabs(z[i]) > amax) amax = fabs(z[i]);
            }
            double sb;
            uint8_t sbyte = e4m3_encode_pos(amax / 6.0, &sb);
            bscale[(size_t)r * nb + b] = sbyte;
            for (int i = 0; i < 16; i += 2) {
                uint8_t lo = sb > 0 ? e2m1_encode(z[i] / sb) : 0;
                uint8_t hi = sb > 0 ? e2m1_encode(z[i + 1] / sb) : 0;
                codes[(size_t)r * (K / 2) + 8 * b + i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* exported for the generator's own tests */
uint16_t synth_half_from_double(double v) { return f64_to_half_rne(v); }
uint8_t synth_e4m3_from_double(double v, double *rounded) { return e4m3_encode_pos(v, rounded); }
uint8_t synth_e2m1_from_double(double v) { return e2m1_encode(v); }
