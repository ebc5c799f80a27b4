/*
 * Device twin of the seeded synthetic-input generator (see wl_gen.h): fills a
 * tensor directly in HBM so full-size layer stacks never pass through the host.
 * Built with --fmad=false so no multiply-add is contracted and every fp64
 * operation rounds as in the host twin.
 */
#include "wl_gen.h"
#include <cuda_runtime.h>

__global__ void wl_fill_kernel(uint64_t seed, uint64_t stream, uint64_t e0, int64_t count,
                               double scale, int bf16, uint16_t* __restrict__ out)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (; i < count; i += stride) out[i] = wl_elem(seed, stream, e0 + (uint64_t)i, scale, bf16);
}

__global__ void wl_row_stats_kernel(const uint16_t* __restrict__ w, int64_t rows, int64_t cols,
                                    int bf16, double* __restrict__ s1, double* __restrict__ s2)
{
    int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const uint16_t* p = w + r * cols;
    double a = 0.0, b = 0.0;
    for (int64_t c = 0; c < cols; ++c) {
        double v = bf16 ? wl_bf16_to_f64(p[c]) : wl_f16_to_f64(p[c]);
        a = __dadd_rn(a, v);
        b = __dadd_rn(b, __dmul_rn(v, v));
    }
    s1[r] = a; s2[r] = b;
}

extern "C" int wl_dev_fill(uint64_t seed, uint64_t stream, uint64_t e0, int64_t count, double scale,
                           int bf16, void* out, void* cuda_stream)
{
    if (count <= 0) return 0;
    int64_t blocks = (count + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    wl_fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(
        seed, stream, e0, count, scale, bf16, (uint16_t*)out);
    return (int)cudaGetLastError();
}

extern "C" int wl_dev_row_stats(const void* w, int64_t rows, int64_t cols, int bf16,
                                double* s1, double* s2, void* cuda_stream)
{
    if (rows <= 0) return 0;
    wl_row_stats_kernel<<<(unsigned)((rows + 127) / 128), 128, 0, (cudaStream_t)cuda_stream>>>(
        (const uint16_t*)w, rows, cols, bf16, s1, s2);
    return (int)cudaGetLastError();
}
