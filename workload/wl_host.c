/*
 * Host twin of the seeded synthetic-input generator (see wl_gen.h).
 * Compiled with -ffp-contract=off so every fp64 operation rounds exactly as
 * written; the device twin (wl_device.cu) uses explicitly rounded intrinsics
 * for the same operations, so both produce identical bits.
 */
#include "wl_gen.h"
#include <stddef.h>

void wl_philox(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    wl_u32x4 o = wl_philox4x32_10(ctr[0], ctr[1], ctr[2], ctr[3], key[0], key[1]);
    for (int i = 0; i < 4; ++i) out[i] = o.v[i];
}

/* out[i] = N(0,1) sample of element e0+i (fp64, unrounded). */
void wl_normal_f64(uint64_t seed, uint64_t stream, uint64_t e0, int64_t count, double* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) out[i] = wl_normal(seed, stream, e0 + (uint64_t)i);
}

/* out[i] = dtype bits of scale * N(0,1) for element e0+i. */
void wl_fill(uint64_t seed, uint64_t stream, uint64_t e0, int64_t count, double scale,
             int bf16, uint16_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) out[i] = wl_elem(seed, stream, e0 + (uint64_t)i, scale, bf16);
}

/* Selected rows of a row-major [*, cols] tensor: out[r][c] = element rows[r]*cols + c. */
void wl_fill_rows(uint64_t seed, uint64_t stream, int64_t cols, const int64_t* rows,
                  int64_t nrows, double scale, int bf16, uint16_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        uint64_t base = (uint64_t)rows[r] * (uint64_t)cols;
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = wl_elem(seed, stream, base + (uint64_t)c, scale, bf16);
    }
}

/* Per-row fp64 sums of w and w*w, summed strictly left to right. */
void wl_row_stats(const uint16_t* w, int64_t rows, int64_t cols, int bf16, double* s1, double* s2)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double a = 0.0, b = 0.0;
        const uint16_t* p = w + r * cols;
        for (int64_t c = 0; c < cols; ++c) {
            double v = bf16 ? wl_bf16_to_f64(p[c]) : wl_f16_to_f64(p[c]);
            a = a + v;
            b = b + v * v;
        }
        s1[r] = a; s2[r] = b;
    }
}

/* Vector rounding helpers (used for biases computed on the host). */
void wl_round_f64(const double* x, int64_t count, int bf16, uint16_t* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = bf16 ? wl_f64_to_bf16(x[i]) : wl_f64_to_f16(x[i]);
}

void wl_widen(const uint16_t* x, int64_t count, int bf16, double* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = bf16 ? wl_bf16_to_f64(x[i]) : wl_f16_to_f64(x[i]);
}

/* 64-bit keys for a seeded shuffle: key[i] = high 64 bits of Philox block i. */
void wl_u64_keys(uint64_t seed, uint64_t stream, int64_t count, uint64_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        wl_u32x4 o = wl_philox4x32_10((uint32_t)i, (uint32_t)((uint64_t)i >> 32),
                                      (uint32_t)stream, (uint32_t)(stream >> 32),
                                      (uint32_t)seed, (uint32_t)(seed >> 32));
        out[i] = ((uint64_t)o.v[0] << 32) | (uint64_t)o.v[1];
    }
}
