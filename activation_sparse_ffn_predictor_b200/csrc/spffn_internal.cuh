// Internal definitions shared by the spffn kernels and the C-ABI glue.
#pragma once
#include <algorithm>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include "../../include/spffn.h"

namespace spffn {

// Device error word bits (latched with atomicOr, read by spffn_last_device_error).
enum : uint32_t {
    ERR_COUNT_CLAMPED = 1u << 0,   // caller-supplied count > n (clamped to n) or < 0 (clamped to 0)
    ERR_IDX_RANGE = 1u << 1,       // a neuron table entry outside [0, n) (skipped)
    ERR_BARRIER_TIMEOUT = 1u << 2, // a grid barrier wait hit its iteration limit
    ERR_PIPE_TIMEOUT = 1u << 3,    // a copy-completion wait hit its iteration limit
    ERR_CACHE_FULL = 1u << 4,      // head-sparse attention: a step found the KV cache full
};

constexpr int kMaxBatch = 256;       // union tensor-core path (B >= 16, d % 128 == 0)
constexpr int kUStackMinBatch = 3;   // whole-stack union kernel: 3 <= B <= 128 (smaller B: the small-batch kernel)
constexpr int kMaxPhaseBatch = 32;   // per-phase kernels and the split-FFN partial buffer
constexpr int kCtlBytes = 1024;    // control block at the head of the workspace
constexpr int kMaxUnionCtas = 256;  // union path: split-K partial capacity in CTAs
constexpr int kUnionTickets = 2048;

// Control block (u32 words) at the start of every workspace.
struct Ctl {
    uint32_t err;          // latched error bits
    uint32_t ticket;       // reserved
    uint32_t pad0[14];
    uint32_t barrier[64];  // persistent kernels: [0] grid barrier, [1] abort of the small-batch decode;
                           // [2], [3] the same for the whole-stack union kernel
};

struct Layout {
    size_t ctl, h, mask, partial, xbuf, ybuf, idx, count, ctacnt, hsplit, asplit, upartial, utickets, uss, utab, total;
    int S;  // number of FFN partial sums
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline Layout make_layout(const spffn_config& c, int S) {
    Layout L;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
    L.S = S;
    L.ctl = take(kCtlBytes);
    // two buffers: the small-batch decode alternates them by predictor layer, so a CTA can
    // write the next layer's h while slower CTAs still read this one (look-ahead prologue)
    L.h = take((size_t)2 * std::max(c.max_batch, 2) * c.H * sizeof(float));
    L.mask = take((size_t)(c.n / 32) * sizeof(uint32_t));
    const int pb = c.max_batch < kMaxPhaseBatch ? c.max_batch : kMaxPhaseBatch;
    L.partial = take((size_t)S * pb * c.d * sizeof(float));
    L.xbuf = take((size_t)2 * c.max_batch * c.d * 2);
    L.ybuf = take((size_t)c.max_batch * c.d * sizeof(float));
    L.idx = take((size_t)c.n * sizeof(int32_t));
    L.count = take(256);
    L.ctacnt = take((size_t)2 * (S + 1) * sizeof(int32_t));    // two lists' per-CTA lengths
    // hi/lo activation rows of the union path: token groups of at most 128 (padded to 16)
    const int srows = 2 * (c.max_batch <= 128 ? (c.max_batch + 15) / 16 * 16 : (c.max_batch + 127) / 128 * 128);
    L.hsplit = take((size_t)srows * c.H * 2);
    L.asplit = take((size_t)srows * c.n * 2);
    if (c.max_batch >= kUStackMinBatch) {
        const int nmax = c.max_batch > 32 ? 256 : 64;    // widest MMA N of a union launch
        L.upartial = take((size_t)kMaxUnionCtas * 128 * nmax * sizeof(float));
        L.utickets = take((size_t)kUnionTickets * sizeof(uint32_t));
        // whole-stack union kernel: per 128-column tile, per token sums of squares of x + y
        L.uss = take((size_t)((c.d + 127) / 128) * c.max_batch * sizeof(float));
        // and every CTA's private copy of the neuron table (no grid barrier before the gathers)
        L.utab = take((size_t)S * c.n * sizeof(int32_t));
    } else {
        L.upartial = L.utickets = L.uss = L.utab = 0;
    }
    L.total = off;
    return L;
}

}  // namespace spffn

struct spffn_ctx {
    spffn_config cfg;
    spffn_weights w;
    char* ws;
    size_t ws_bytes;
    spffn::Layout lay;
    int num_sms;
    int device;

    spffn::Ctl* ctl() const { return reinterpret_cast<spffn::Ctl*>(ws + lay.ctl); }
    float* h() const { return reinterpret_cast<float*>(ws + lay.h); }
    uint32_t* mask() const { return reinterpret_cast<uint32_t*>(ws + lay.mask); }
    float* partial() const { return reinterpret_cast<float*>(ws + lay.partial); }
    void* xbuf(int i) const { return ws + lay.xbuf + (size_t)i * cfg.max_batch * cfg.d * 2; }
    float* ybuf() const { return reinterpret_cast<float*>(ws + lay.ybuf); }
    int32_t* idx() const { return reinterpret_cast<int32_t*>(ws + lay.idx); }
    int32_t* count() const { return reinterpret_cast<int32_t*>(ws + lay.count); }
    int32_t* ctacnt() const { return reinterpret_cast<int32_t*>(ws + lay.ctacnt); }
    void* hsplit() const { return ws + lay.hsplit; }
    void* asplit() const { return ws + lay.asplit; }
    float* upartial() const { return reinterpret_cast<float*>(ws + lay.upartial); }
    uint32_t* utickets() const { return reinterpret_cast<uint32_t*>(ws + lay.utickets); }
    float* uss() const { return reinterpret_cast<float*>(ws + lay.uss); }
    int32_t* utab() const { return reinterpret_cast<int32_t*>(ws + lay.utab); }
};

namespace spffn {

// ---------------------------------------------------------------------------
// storage-dtype helpers
template <typename T> struct DT;
template <> struct DT<__half> {
    static __device__ __forceinline__ float f(__half v) { return __half2float(v); }
    static __device__ __forceinline__ __half r(float v) { return __float2half_rn(v); }
    static __device__ __forceinline__ float2 f2(uint32_t u) {
        __half2 h = *reinterpret_cast<__half2*>(&u);
        return __half22float2(h);
    }
};
template <> struct DT<__nv_bfloat16> {
    static __device__ __forceinline__ float f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 r(float v) { return __float2bfloat16_rn(v); }
    static __device__ __forceinline__ float2 f2(uint32_t u) {
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
        return __bfloat1622float2(h);
    }
};

// 8 storage elements (one 16-byte vector) -> 8 floats
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
    float2 a = DT<T>::f2(v.x), b = DT<T>::f2(v.y), c = DT<T>::f2(v.z), d = DT<T>::f2(v.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void latch(uint32_t* err, uint32_t bits) { atomicOr(err, bits); }

}  // namespace spffn
