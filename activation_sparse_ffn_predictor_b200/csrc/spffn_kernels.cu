// Per-phase kernels of the sparse-FFN decode path (one launch per phase).
//
// These serve spffn_predict and spffn_forward at batches 3..15 (and for shapes
// outside the persistent kernel's limits; batches of 16 and more run on the union
// path, and spffn_forward at 1..2 on the persistent kernel), spffn_chain, and the
// offline profile and permutation calls.  Every weight row is read with 16-byte
// vector loads that bypass L1 (each row is touched once per call); fp32
// accumulation throughout; every reduction has a fixed order.
#include "spffn_internal.cuh"
#include "spffn_kernels.cuh"
#include "spffn_union.cuh"

namespace spffn {

// programmatic dependent launch (no-ops when the launch has no programmatic dependency)
__device__ __forceinline__ void pdl_trigger_k() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_k() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

static cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, cudaStream_t st, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// ---------------------------------------------------------------------------
// S1  predictor hidden layer: h[t][r] = ReLU(Wp1[r] . x_t + bp1[r])
// One warp per predictor row; tokens in groups of 8 held in registers.
template <typename T>
__global__ void __launch_bounds__(256) k_hidden(const T* __restrict__ Wp1, const T* __restrict__ bp1,
                                                const T* __restrict__ x, int B, int d, int H,
                                                float* __restrict__ h)
{
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int nw = gridDim.x * (blockDim.x >> 5);
    const int nv = d >> 3;
    for (int r = gw; r < H; r += nw) {
        const uint4* wrow = reinterpret_cast<const uint4*>(Wp1 + (size_t)r * d);
        const float bias = bp1 ? DT<T>::f(bp1[r]) : 0.f;
        for (int t0 = 0; t0 < B; t0 += 8) {
            const int nt = min(8, B - t0);
            float acc[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[t] = 0.f;
            auto fold = [&](const uint4& wv, int v) {
                float w[8];
                unpack8<T>(wv, w);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (t < nt) {
                        float xv[8];
                        unpack8<T>(__ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * d) + v), xv);
#pragma unroll
                        for (int k = 0; k < 8; ++k) acc[t] = fmaf(w[k], xv[k], acc[t]);
                    }
                }
            };
            // four weight vectors per lane in flight before they are used (the loads are
            // volatile asm, which the compiler does not move across each other)
            int v = lane;
            for (; v + 96 < nv; v += 128) {
                const uint4 w0 = ldg_stream(wrow + v), w1 = ldg_stream(wrow + v + 32);
                const uint4 w2 = ldg_stream(wrow + v + 64), w3 = ldg_stream(wrow + v + 96);
                fold(w0, v); fold(w1, v + 32); fold(w2, v + 64); fold(w3, v + 96);
            }
            for (; v < nv; v += 32) fold(ldg_stream(wrow + v), v);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (t < nt) {
                    float s = warp_sum(acc[t]);
                    if (lane == 0) h[(size_t)(t0 + t) * H + r] = fmaxf(s + bias, 0.f);
                }
            }
        }
    }
}

// The same layer for B <= 8 with each row split over four warps of one CTA (two rows
// per CTA): four times the warps streaming Wp1, so a 1-8 token GEMV keeps enough
// loads in flight to cover HBM latency.  The four quarter sums are added in a fixed
// order.
template <typename T>
__global__ void __launch_bounds__(256) k_hidden_split(const T* __restrict__ Wp1, const T* __restrict__ bp1,
                                                      const T* __restrict__ x, int B, int d, int H,
                                                      float* __restrict__ h)
{
    __shared__ float part[8][8];                        // [warp][token]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = blockIdx.x * 2 + (warp >> 2), q = warp & 3;
    const int nv = d >> 3, v0 = nv * q / 4, v1 = nv * (q + 1) / 4;
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
    if (r < H) {
        const uint4* wrow = reinterpret_cast<const uint4*>(Wp1 + (size_t)r * d);
        auto fold = [&](const uint4& wv, int v) {
            float w[8];
            unpack8<T>(wv, w);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (t < B) {
                    float xv[8];
                    unpack8<T>(__ldg(reinterpret_cast<const uint4*>(x + (size_t)t * d) + v), xv);
#pragma unroll
                    for (int k = 0; k < 8; ++k) acc[t] = fmaf(w[k], xv[k], acc[t]);
                }
            }
        };
        int v = v0 + lane;
        for (; v + 96 < v1; v += 128) {
            const uint4 w0 = ldg_stream(wrow + v), w1 = ldg_stream(wrow + v + 32);
            const uint4 w2 = ldg_stream(wrow + v + 64), w3 = ldg_stream(wrow + v + 96);
            fold(w0, v); fold(w1, v + 32); fold(w2, v + 64); fold(w3, v + 96);
        }
        for (; v < v1; v += 32) fold(ldg_stream(wrow + v), v);
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const float sum = warp_sum(acc[t]);
        if (lane == 0) part[warp][t] = sum;
    }
    __syncthreads();
    if (threadIdx.x < 2 * B) {
        const int rr = threadIdx.x / B, t = threadIdx.x - rr * B, row = blockIdx.x * 2 + rr;
        if (row < H) {
            const float* pr = &part[rr * 4][0];
            const float sum = (pr[t] + pr[8 + t]) + (pr[16 + t] + pr[24 + t]);
            const float bias = bp1 ? DT<T>::f(bp1[row]) : 0.f;
            h[(size_t)t * H + row] = fmaxf(sum + bias, 0.f);
        }
    }
}

// ---------------------------------------------------------------------------
// S2  predictor output layer + threshold: neuron i selected iff some token has
// Wp2[i] . h_t + bp2[i] > 0.  A block of 8 warps owns one 32-neuron word.
template <typename T>
__global__ void __launch_bounds__(256) k_logits(const T* __restrict__ Wp2, const T* __restrict__ bp2,
                                                const float* __restrict__ h, int B, int H, int n,
                                                uint32_t* __restrict__ mask)
{
    __shared__ int sel[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nv = H >> 3;
    for (int word = blockIdx.x; word < (n >> 5); word += gridDim.x) {
        for (int q = warp; q < 32; q += 8) {
            const int row = word * 32 + q;
            const uint4* wrow = reinterpret_cast<const uint4*>(Wp2 + (size_t)row * H);
            const float bias = bp2 ? DT<T>::f(bp2[row]) : 0.f;
            bool any = false;
            for (int t0 = 0; t0 < B; t0 += 8) {
                const int nt = min(8, B - t0);
                float acc[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) acc[t] = 0.f;
                for (int v = lane; v < nv; v += 32) {
                    float w[8];
                    unpack8<T>(ldg_stream(wrow + v), w);
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        if (t < nt) {
                            const float4* hp = reinterpret_cast<const float4*>(h + (size_t)(t0 + t) * H) + 2 * v;
                            float4 a = __ldg(hp), b = __ldg(hp + 1);
                            acc[t] = fmaf(w[0], a.x, acc[t]); acc[t] = fmaf(w[1], a.y, acc[t]);
                            acc[t] = fmaf(w[2], a.z, acc[t]); acc[t] = fmaf(w[3], a.w, acc[t]);
                            acc[t] = fmaf(w[4], b.x, acc[t]); acc[t] = fmaf(w[5], b.y, acc[t]);
                            acc[t] = fmaf(w[6], b.z, acc[t]); acc[t] = fmaf(w[7], b.w, acc[t]);
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    if (t < nt) any |= (warp_sum(acc[t]) + bias) > 0.f;
            }
            if (lane == 0) sel[q] = any ? 1 : 0;
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t bits = __ballot_sync(0xffffffffu, sel[lane] != 0);
            if (lane == 0) mask[word] = bits;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// S3  compaction: ascending neuron table from the mask words.  One block of
// 1024 threads; thread q owns words [q*per, (q+1)*per).
__global__ void __launch_bounds__(1024) k_compact(const uint32_t* __restrict__ mask, int words,
                                                  int32_t* __restrict__ idx, int32_t* __restrict__ count,
                                                  int32_t* __restrict__ count2)
{
    __shared__ uint32_t wsum[32];
    pdl_trigger_k();
    pdl_wait_k();                                  // the mask words come from the previous kernel
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (words + 1023) / 1024;
    const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
    uint32_t local = 0;
    for (int w = w0; w < w1; ++w) local += __popc(mask[w]);
    // inclusive warp scan
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t v = wsum[lane];
        uint32_t s = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t u = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += u;
        }
        wsum[lane] = s - v;  // exclusive prefix of warp totals
        if (lane == 31) { *count = (int32_t)s; if (count2) *count2 = (int32_t)s; }
    }
    __syncthreads();
    uint32_t pos = wsum[warp] + incl - local;
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = mask[w];
        while (bits) {
            int b = __ffs(bits) - 1;
            bits &= bits - 1;
            idx[pos++] = w * 32 + b;
        }
    }
}

// ---------------------------------------------------------------------------
// S4+S5  neuron-aware FFN, stage 1: CTA s takes table entries
// [s*k/S, (s+1)*k/S) and accumulates  sum_j ReLU(W1[j].x_t + b1_j) W2T[j]
// into fp32 partial[s][t][:].  Each thread owns fixed 8-column vectors, so the
// per-column accumulation order is the table order (deterministic).
template <typename T>
__global__ void __launch_bounds__(256) k_ffn_partial(const T* __restrict__ W1, const T* __restrict__ b1,
                                                     const T* __restrict__ W2T, const T* __restrict__ x,
                                                     int B, int d, int n, const int32_t* __restrict__ idx,
                                                     const int32_t* __restrict__ count, int tg,
                                                     float* __restrict__ partial, uint32_t* __restrict__ err)
{
    extern __shared__ float acc[];           // [tg][d]
    __shared__ float red[2][8][8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nv = d >> 3;
    int k = *count;
    if (k > n || k < 0) {
        if (blockIdx.x == 0 && tid == 0) latch(err, ERR_COUNT_CLAMPED);
        k = k < 0 ? 0 : n;
    }
    const int S = gridDim.x, s = blockIdx.x;
    const int lo = (int)((long long)s * k / S), hi = (int)((long long)(s + 1) * k / S);
    int parity = 0;
    for (int t0 = 0; t0 < B; t0 += tg) {
        const int nt = min(tg, B - t0);
        for (int i = tid; i < nt * d; i += blockDim.x) acc[i] = 0.f;
        __syncthreads();
        for (int pos = lo; pos < hi; ++pos) {
            const int j = idx[pos];
            if (j < 0 || j >= n) {
                if (tid == 0) latch(err, ERR_IDX_RANGE);
                continue;
            }
            const uint4* w1 = reinterpret_cast<const uint4*>(W1 + (size_t)j * d);
            const uint4* w2 = reinterpret_cast<const uint4*>(W2T + (size_t)j * d);
            float part[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) part[t] = 0.f;
            for (int v = tid; v < nv; v += blockDim.x) {
                float w[8];
                unpack8<T>(ldg_stream(w1 + v), w);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (t < nt) {
                        float xv[8];
                        unpack8<T>(__ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * d) + v), xv);
#pragma unroll
                        for (int q = 0; q < 8; ++q) part[t] = fmaf(w[q], xv[q], part[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                float v = warp_sum(part[t]);
                if (lane == 0) red[parity][warp][t] = v;
            }
            __syncthreads();
            const float bias = DT<T>::f(b1[j]);
            float a[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                float z = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) z += red[parity][q][t];
                a[t] = fmaxf(z + bias, 0.f);
            }
            parity ^= 1;
            for (int v = tid; v < nv; v += blockDim.x) {
                float w[8];
                unpack8<T>(ldg_stream(w2 + v), w);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (t < nt) {
                        float* ap = acc + (size_t)t * d + v * 8;
#pragma unroll
                        for (int q = 0; q < 8; ++q) ap[q] = fmaf(a[t], w[q], ap[q]);
                    }
                }
            }
        }
        __syncthreads();
        for (int i = tid; i < nt * d; i += blockDim.x) {
            const int t = i / d, c = i - t * d;
            partial[((size_t)s * B + t0 + t) * d + c] = acc[i];
        }
        __syncthreads();
    }
}

// S6  stage 2: y[t][c] = b2[c] + sum_{s=0..S-1} partial[s][t][c], fixed order.
template <typename T>
__global__ void __launch_bounds__(256) k_ffn_reduce(const float* __restrict__ partial, int S, int B, int d,
                                                    const T* __restrict__ b2, float* __restrict__ y)
{
    const int t = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= d) return;
    float v = 0.f;
    for (int s = 0; s < S; ++s) v += partial[((size_t)s * B + t) * d + c];
    y[(size_t)t * d + c] = v + (b2 ? DT<T>::f(b2[c]) : 0.f);
}

// ---------------------------------------------------------------------------
// S9  chaining: x_next = round((x + y) / sqrt(mean((x + y)^2) + eps)), one block
// of 1024 threads per token; each thread keeps its 8-column vectors of u in
// registers between the sum of squares and the write (fixed reduction tree).
template <typename T>
__global__ void __launch_bounds__(1024) k_chain(const T* __restrict__ x, const float* __restrict__ y, int d,
                                                T* __restrict__ xn)
{
    constexpr int kV = 2;                         // 8-column vectors per thread (d <= 16384)
    __shared__ float ws[32];
    pdl_trigger_k();
    pdl_wait_k();                                 // y comes from the previous kernel
    const int t = blockIdx.x, tid = threadIdx.x;
    const int nv = d >> 3;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    const float4* yr = reinterpret_cast<const float4*>(y + (size_t)t * d);
    float u[kV][8];
    float ss = 0.f;
#pragma unroll
    for (int m = 0; m < kV; ++m) {
        const int v = tid + m * 1024;
        if (v < nv) {
            float xv[8];
            unpack8<T>(xr[v], xv);
            const float4 a = yr[2 * v], b = yr[2 * v + 1];
            const float yv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                u[m][q] = xv[q] + yv[q];
                ss = fmaf(u[m][q], u[m][q], ss);
            }
        }
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) ws[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q) tot += ws[q];
    const float rs = 1.0f / sqrtf(tot / (float)d + 1e-6f);
#pragma unroll
    for (int m = 0; m < kV; ++m) {
        const int v = tid + m * 1024;
        if (v < nv) {
            T o[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) o[q] = DT<T>::r(u[m][q] * rs);
            reinterpret_cast<uint4*>(xn + (size_t)t * d)[v] = *reinterpret_cast<const uint4*>(o);
        }
    }
}

// ---------------------------------------------------------------------------
// S8  offline profile: counts[j] += #{t : W1[j].X_t + b1_j > 0}; one warp per row.
template <typename T>
__global__ void __launch_bounds__(256) k_profile(const T* __restrict__ W1, const T* __restrict__ b1,
                                                 const T* __restrict__ X, int T_, int d, int n,
                                                 uint32_t* __restrict__ counts)
{
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int nw = gridDim.x * (blockDim.x >> 5);
    const int nv = d >> 3;
    for (int j = gw; j < n; j += nw) {
        const uint4* wrow = reinterpret_cast<const uint4*>(W1 + (size_t)j * d);
        const float bias = DT<T>::f(b1[j]);
        uint32_t c = 0;
        for (int t0 = 0; t0 < T_; t0 += 8) {
            const int nt = min(8, T_ - t0);
            float acc[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[t] = 0.f;
            for (int v = lane; v < nv; v += 32) {
                float w[8];
                unpack8<T>(__ldg(wrow + v), w);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (t < nt) {
                        float xv[8];
                        unpack8<T>(__ldg(reinterpret_cast<const uint4*>(X + (size_t)(t0 + t) * d) + v), xv);
#pragma unroll
                        for (int q = 0; q < 8; ++q) acc[t] = fmaf(w[q], xv[q], acc[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 8; ++t)
                if (t < nt) c += (warp_sum(acc[t]) + bias) > 0.f;
        }
        if (lane == 0) counts[j] += c;
    }
}

__global__ void k_permute_rows(const uint4* __restrict__ src, uint4* __restrict__ dst, int rows, int vpr,
                               const int32_t* __restrict__ perm)
{
    for (int s = blockIdx.x; s < rows; s += gridDim.x) {
        const int r = perm[s];
        if (r < 0 || r >= rows) continue;
        for (int v = threadIdx.x; v < vpr; v += blockDim.x)
            dst[(size_t)s * vpr + v] = src[(size_t)r * vpr + v];
    }
}

__global__ void k_permute_vec(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int count,
                              const int32_t* __restrict__ perm)
{
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s < count) {
        const int r = perm[s];
        if (r >= 0 && r < count) dst[s] = src[r];
    }
}

// ---------------------------------------------------------------------------
// launchers
template <typename T>
static cudaError_t predict_impl(const spffn_ctx& c, const void* x, int B, int32_t* idx, int32_t* count,
                                int32_t* count2, cudaStream_t st)
{
    const auto& g = c.cfg;
    const cudaError_t e = launch_hidden(g.dtype, c.w.Wp1, c.w.bp1, x, B, g.d, g.H, c.h(), c.num_sms, st);
    if (e != cudaSuccess) return e;
    const int words = g.n / 32;
    k_logits<T><<<words, 256, 0, st>>>((const T*)c.w.Wp2, (const T*)c.w.bp2, c.h(), B, g.H, g.n, c.mask());
    k_compact<<<1, 1024, 0, st>>>(c.mask(), words, idx, count, count2);
    return cudaGetLastError();
}

int ffn_token_group(const spffn_ctx& c)
{
    // tokens whose fp32 accumulators fit the dynamic shared memory budget
    const int budget = 160 * 1024;
    int tg = budget / (c.cfg.d * (int)sizeof(float));
    return max(1, min(8, tg));
}

template <typename T>
static cudaError_t forward_impl(const spffn_ctx& c, const void* x, int B, const int32_t* idx,
                                const int32_t* count, float* y, cudaStream_t st)
{
    const auto& g = c.cfg;
    const int tg = ffn_token_group(c);
    const size_t smem = (size_t)tg * g.d * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k_ffn_partial<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_ffn_partial<T><<<c.lay.S, 256, smem, st>>>((const T*)c.w.W1, (const T*)c.w.b1, (const T*)c.w.W2T,
                                                 (const T*)x, B, g.d, g.n, idx, count, tg, c.partial(),
                                                 &c.ctl()->err);
    dim3 rg((g.d + 255) / 256, B);
    k_ffn_reduce<T><<<rg, 256, 0, st>>>(c.partial(), c.lay.S, B, g.d, (const T*)c.w.b2, y);
    return cudaGetLastError();
}

// Same two kernels as forward_impl, with caller-chosen scratch (S partial sums
// of B x d fp32 at `partial`, error word at `err`).
template <typename T>
static cudaError_t forward_scratch_impl(const spffn_config& g, const spffn_weights& w, const void* x, int B,
                                        const int32_t* idx, const int32_t* count, float* y, float* partial, int S,
                                        uint32_t* err, cudaStream_t st)
{
    const int tg = max(1, min(8, (160 * 1024) / (g.d * (int)sizeof(float))));
    const size_t smem = (size_t)tg * g.d * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k_ffn_partial<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_ffn_partial<T><<<S, 256, smem, st>>>((const T*)w.W1, (const T*)w.b1, (const T*)w.W2T, (const T*)x, B, g.d, g.n,
                                           idx, count, tg, partial, err);
    dim3 rg((g.d + 255) / 256, B);
    k_ffn_reduce<T><<<rg, 256, 0, st>>>(partial, S, B, g.d, (const T*)w.b2, y);
    return cudaGetLastError();
}

cudaError_t launch_forward_scratch(const spffn_config& g, const spffn_weights& w, const void* x, int B,
                                   const int32_t* idx, const int32_t* count, float* y, float* partial, int S,
                                   uint32_t* err, cudaStream_t st)
{
    return g.dtype == SPFFN_BF16
               ? forward_scratch_impl<__nv_bfloat16>(g, w, x, B, idx, count, y, partial, S, err, st)
               : forward_scratch_impl<__half>(g, w, x, B, idx, count, y, partial, S, err, st);
}

template <typename T>
static cudaError_t chain_impl(const spffn_ctx& c, const void* x, const float* y, int B, void* xn, cudaStream_t st)
{
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = pdl_config(dim3(B), dim3(1024), st, attr);
    return cudaLaunchKernelEx(&cfg, k_chain<T>, (const T*)x, y, c.cfg.d, (T*)xn);
}

template <typename T>
static cudaError_t profile_impl(const spffn_ctx& c, const void* X, int T_, uint32_t* counts, cudaStream_t st)
{
    const int blocks = min((c.cfg.n + 7) / 8, c.num_sms * 8);
    k_profile<T><<<blocks, 256, 0, st>>>((const T*)c.w.W1, (const T*)c.w.b1, (const T*)X, T_, c.cfg.d, c.cfg.n,
                                         counts);
    return cudaGetLastError();
}

cudaError_t launch_hidden(int dtype, const void* W, const void* b, const void* x, int B, int d, int H, float* h,
                          int num_sms, cudaStream_t st)
{
    if (B <= 8) {
        const int hb2 = (H + 1) / 2;
        if (dtype == SPFFN_BF16)
            k_hidden_split<__nv_bfloat16><<<hb2, 256, 0, st>>>((const __nv_bfloat16*)W, (const __nv_bfloat16*)b,
                                                               (const __nv_bfloat16*)x, B, d, H, h);
        else
            k_hidden_split<__half><<<hb2, 256, 0, st>>>((const __half*)W, (const __half*)b, (const __half*)x, B, d,
                                                        H, h);
        return cudaGetLastError();
    }
    const int hb = min((H + 7) / 8, num_sms * 8);
    if (dtype == SPFFN_BF16)
        k_hidden<__nv_bfloat16><<<hb, 256, 0, st>>>((const __nv_bfloat16*)W, (const __nv_bfloat16*)b,
                                                    (const __nv_bfloat16*)x, B, d, H, h);
    else
        k_hidden<__half><<<hb, 256, 0, st>>>((const __half*)W, (const __half*)b, (const __half*)x, B, d, H, h);
    return cudaGetLastError();
}

cudaError_t launch_compact(const spffn_ctx& c, int32_t* idx, int32_t* count, int32_t* count2, cudaStream_t st)
{
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = pdl_config(dim3(1), dim3(1024), st, attr);
    return cudaLaunchKernelEx(&cfg, k_compact, (const uint32_t*)c.mask(), c.cfg.n / 32, idx, count, count2);
}

cudaError_t launch_predict(const spffn_ctx& c, const void* x, int B, int32_t* idx, int32_t* count,
                           int32_t* count2, cudaStream_t st, bool defer_table)
{
    if (union_supported(c, B)) return union_predict(c, x, B, idx, count, count2, st, defer_table);
    return c.cfg.dtype == SPFFN_BF16 ? predict_impl<__nv_bfloat16>(c, x, B, idx, count, count2, st)
                                     : predict_impl<__half>(c, x, B, idx, count, count2, st);
}

cudaError_t launch_forward(const spffn_ctx& c, const void* x, int B, const int32_t* idx, const int32_t* count,
                           float* y, cudaStream_t st, int32_t* table_out, int32_t* count2)
{
    if (union_supported(c, B)) return union_forward(c, x, B, idx, count, y, st, table_out, count2);
    return c.cfg.dtype == SPFFN_BF16 ? forward_impl<__nv_bfloat16>(c, x, B, idx, count, y, st)
                                     : forward_impl<__half>(c, x, B, idx, count, y, st);
}

cudaError_t launch_chain(const spffn_ctx& c, const void* x, const float* y, int B, void* xn, cudaStream_t st)
{
    return c.cfg.dtype == SPFFN_BF16 ? chain_impl<__nv_bfloat16>(c, x, y, B, xn, st)
                                     : chain_impl<__half>(c, x, y, B, xn, st);
}

cudaError_t launch_profile(const spffn_ctx& c, const void* X, int T_, uint32_t* counts, cudaStream_t st)
{
    return c.cfg.dtype == SPFFN_BF16 ? profile_impl<__nv_bfloat16>(c, X, T_, counts, st)
                                     : profile_impl<__half>(c, X, T_, counts, st);
}

cudaError_t launch_permute_rows(const void* src, void* dst, int rows, int row_bytes, const int32_t* perm,
                                cudaStream_t st)
{
    const int vpr = row_bytes / 16;
    const int blocks = min(rows, 148 * 16);
    k_permute_rows<<<blocks, 256, 0, st>>>((const uint4*)src, (uint4*)dst, rows, vpr, perm);
    return cudaGetLastError();
}

cudaError_t launch_permute_vec(const void* src, void* dst, int count, const int32_t* perm, cudaStream_t st)
{
    k_permute_vec<<<(count + 255) / 256, 256, 0, st>>>((const uint16_t*)src, (uint16_t*)dst, count, perm);
    return cudaGetLastError();
}

}  // namespace spffn
