/*
 * Seeded synthetic inputs: one counter-based generator, compiled for the host
 * (wl_host.c) and for the device (wl_device.cu) from this single definition, so
 * that a tensor filled on either side holds the same bits.
 *
 * This file holds no arithmetic of the sparse-FFN method itself: only random
 * numbers, their scaling, rounding to the storage dtype, and the fp64 row sums
 * used to calibrate biases.
 *
 *  - Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *    easy as 1, 2, 3", SC'11.  Ten rounds of the 4x32 bijection with multipliers
 *    0xD2511F53 / 0xCD9E8D57 and Weyl key increments 0x9E3779B9 / 0xBB67AE85.
 *  - Box-Muller transform (Box & Muller 1958) on two 53-bit uniforms in (0,1).
 *  - Round-to-nearest-even from fp64 to IEEE binary16 / bfloat16 by integer
 *    manipulation of the fp64 bit pattern (no library conversion).
 *
 * Element e of a tensor (row-major flat index) uses Philox block e>>1 and the
 * first (even e) or second (odd e) normal of that block.  The counter is
 * (block_lo, block_hi, stream_lo, stream_hi), the key is the 64-bit seed.
 */
#ifndef WL_GEN_H
#define WL_GEN_H
#include <stdint.h>
#include <math.h>

#ifdef __CUDACC__
#define WL_HD __host__ __device__ __forceinline__
#else
#define WL_HD static inline
#endif

typedef struct { uint32_t v[4]; } wl_u32x4;

WL_HD wl_u32x4 wl_philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                uint32_t k0, uint32_t k1)
{
    for (int r = 0; r < 10; ++r) {
        if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    }
    wl_u32x4 o; o.v[0] = c0; o.v[1] = c1; o.v[2] = c2; o.v[3] = c3;
    return o;
}

/* 53-bit uniform strictly inside (0,1): (m + 0.5) * 2^-53, m in [0, 2^53). */
WL_HD double wl_u53(uint32_t hi, uint32_t lo)
{
    uint64_t m = (((uint64_t)hi << 32) | (uint64_t)lo) >> 11;
    return ((double)m + 0.5) * 1.1102230246251565e-16; /* 2^-53 */
}

/* Standard normal for flat element e of the stream `stream` under `seed`. */
WL_HD double wl_normal(uint64_t seed, uint64_t stream, uint64_t e)
{
    uint64_t b = e >> 1;
    wl_u32x4 o = wl_philox4x32_10((uint32_t)b, (uint32_t)(b >> 32),
                                  (uint32_t)stream, (uint32_t)(stream >> 32),
                                  (uint32_t)seed, (uint32_t)(seed >> 32));
    double u1 = wl_u53(o.v[0], o.v[1]);
    double u2 = wl_u53(o.v[2], o.v[3]);
    double r = sqrt(-2.0 * log(u1));
    double t = 6.283185307179586 * u2;
    return (e & 1) ? r * sin(t) : r * cos(t);
}

/* fp64 -> binary16 bits, round to nearest even, with subnormals and overflow. */
WL_HD uint16_t wl_f64_to_f16(double x)
{
    union { double d; uint64_t u; } c; c.d = x;
    uint64_t u = c.u;
    uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
    int64_t e = (int64_t)((u >> 52) & 0x7FF);
    uint64_t m = u & 0xFFFFFFFFFFFFFull;
    if (e == 0x7FF) return (uint16_t)(sign | 0x7C00u | (m ? 0x200u : 0u));
    int64_t ue = e - 1023;                 /* unbiased exponent */
    if (ue > 15) return (uint16_t)(sign | 0x7C00u);
    uint64_t full = m | (e ? (1ull << 52) : 0ull);  /* 53-bit significand */
    int shift;                             /* bits to drop from `full` */
    uint16_t hexp;
    if (ue >= -14) { shift = 42; hexp = (uint16_t)(ue + 15); }
    else { shift = (int)(42 + (-14 - ue)); hexp = 0; if (shift > 63) return sign; }
    uint64_t keep = full >> shift;
    uint64_t rem = full & ((1ull << shift) - 1ull);
    uint64_t half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (keep & 1ull))) keep += 1ull;
    /* keep holds the 11-bit significand (normal) or the subnormal mantissa. */
    uint32_t bits;
    if (hexp) {
        if (keep >> 11) { keep >>= 1; hexp += 1; }
        if (hexp >= 31) return (uint16_t)(sign | 0x7C00u);
        bits = ((uint32_t)hexp << 10) | (uint32_t)(keep & 0x3FFu);
    } else {
        bits = (uint32_t)keep;             /* may round up into the smallest normal */
    }
    return (uint16_t)(sign | bits);
}

/* fp64 -> bfloat16 bits, round to nearest even (finite inputs). */
WL_HD uint16_t wl_f64_to_bf16(double x)
{
    union { double d; uint64_t u; } c; c.d = x;
    uint64_t u = c.u;
    uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
    int64_t e = (int64_t)((u >> 52) & 0x7FF);
    uint64_t m = u & 0xFFFFFFFFFFFFFull;
    if (e == 0x7FF) return (uint16_t)(sign | 0x7F80u | (m ? 0x40u : 0u));
    int64_t ue = e - 1023;
    if (ue > 127) return (uint16_t)(sign | 0x7F80u);
    uint64_t full = m | (e ? (1ull << 52) : 0ull);
    int shift;
    uint32_t bexp;
    if (ue >= -126) { shift = 45; bexp = (uint32_t)(ue + 127); }
    else { shift = (int)(45 + (-126 - ue)); bexp = 0; if (shift > 63) return sign; }
    uint64_t keep = full >> shift;
    uint64_t rem = full & ((1ull << shift) - 1ull);
    uint64_t half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (keep & 1ull))) keep += 1ull;
    uint32_t bits;
    if (bexp) {
        if (keep >> 8) { keep >>= 1; bexp += 1; }
        if (bexp >= 255) return (uint16_t)(sign | 0x7F80u);
        bits = (bexp << 7) | (uint32_t)(keep & 0x7Fu);
    } else {
        bits = (uint32_t)keep;
    }
    return (uint16_t)(sign | bits);
}

/* Storage-bits -> fp64 (exact widening). */
WL_HD double wl_f16_to_f64(uint16_t h)
{
    uint32_t s = h >> 15, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(m | 0x400), (int)e - 25);
    return s ? -v : v;
}

WL_HD double wl_bf16_to_f64(uint16_t h)
{
    union { float f; uint32_t u; } c; c.u = ((uint32_t)h) << 16;
    return (double)c.f;
}

/* One element of a scaled normal tensor, rounded to the storage dtype. */
WL_HD uint16_t wl_elem(uint64_t seed, uint64_t stream, uint64_t e, double scale, int bf16)
{
    double z = wl_normal(seed, stream, e) * scale;
    return bf16 ? wl_f64_to_bf16(z) : wl_f64_to_f16(z);
}

#endif
