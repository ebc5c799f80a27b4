// Head-sparse attention decode with DejaVu's attention-head predictor (SP_A),
// the attention half of equation (-1) in the DejaVu appendix of
// "LLM模型之PowerInfer1.0": S_A <- SP_A(y), y~ <- MHA restricted to S_A, with
// the page's handling of KV-cache misses (a head selected after being skipped
// computes its missing K/V rows from the stored inputs of the past tokens).
//
// One step of one layer, one token, five launches on the caller's stream:
//   1 SP_A hidden layer h = ReLU(Wa1 y + ba1)                 (the predictor GEMV kernel)
//   2 one CTA per head: its logit and decision, and for a selected head the list
//     of positions p < t whose K/V rows are missing; y stored as Y[t]; the CTA
//     finishing last writes the ascending head list and the q/k/v work units
//   3 q, k, v rows of the selected heads for the new token, and the missing K/V
//     rows from Y[p], in work units balanced over every resident warp
//   4 attention per selected head over positions 0..t, split over CTAs with an
//     online softmax in fixed position order, the splits combined in fixed
//     order by the last CTA of the head (atomic ticket)
//   5 out = bo + sum of o_k[i] WoT[k dh + i] over the selected heads' rows, each
//     CTA owning a slice of out's columns (sums in a fixed order); t = t + 1 (the
//     position lives on the device, so a step replays in a CUDA graph)
// Weight bytes dominate (Wa1, the selected heads' Wq/Wk/Wv/Wo rows, then the
// cached K/V rows): every kernel streams rows with 16-byte loads.
#include <algorithm>
#include <cstring>
#include <new>
#include "spffn_internal.cuh"
#include "spffn_kernels.cuh"
#include "../../include/spffn_attn.h"

namespace spffn {

struct ALayout {
    size_t ctl, h, q, miss, nmiss, hsel, upref, opart, o, tickets, K, V, filled, Y, total;
    int S, Sa;
};

inline ALayout attn_layout(const spffn_attn_config& c, int S) {
    ALayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
    L.S = S;
    L.Sa = 8;                                                   // position splits per head
    L.ctl = take(256);                                          // [0] error word, [1] t, [2] select ticket
    L.h = take((size_t)c.Ha * sizeof(float));
    L.q = take((size_t)c.nh * c.dh * sizeof(float));
    L.miss = take((size_t)c.nh * c.tmax * sizeof(uint16_t));    // per head: missing positions
    L.nmiss = take((size_t)c.nh * sizeof(int32_t));
    L.hsel = take((size_t)c.nh * sizeof(int32_t));             // per head: selected this step
    L.upref = take((size_t)(c.nh + 1) * sizeof(int32_t));     // work units before each head slot
    L.opart = take((size_t)c.nh * L.Sa * (c.dh + 2) * sizeof(float));
    L.o = take((size_t)c.nh * c.dh * sizeof(float));
    L.tickets = take((size_t)c.nh * sizeof(uint32_t));
    L.K = take((size_t)c.nh * c.tmax * c.dh * 2);
    L.V = take((size_t)c.nh * c.tmax * c.dh * 2);
    L.filled = take((size_t)c.nh * c.tmax);
    L.Y = take((size_t)c.tmax * c.d * 2);
    L.total = off;
    return L;
}

struct AParams {
    const void *Wq, *bq, *Wk, *bk, *Wv, *bv, *WoT, *bo, *Wa2, *ba2;
    const void* y;
    int d, nh, dh, Ha, tmax, Sa;
    int32_t* tcur;
    int32_t* heads;
    int32_t* count;
    uint32_t* err;
    const float* h;
    float* q;
    uint16_t* miss;
    int32_t* nmiss;
    int32_t* hsel;
    uint32_t* sticket;
    int32_t* upref;
    float* opart;
    float* o;
    uint32_t* tickets;
    void* K;
    void* V;
    uint8_t* filled;
    void* Y;
    float* out;
};

namespace {

constexpr int kPos = 4;                                 // positions per k/v work unit
constexpr int kRW = 4;                                  // weight rows per q/k/v work unit (dh % 8 == 0)

template <typename T>
__device__ __forceinline__ float dot8(const uint4& w, const uint4& x) {
    float a[8], b[8];
    unpack8<T>(w, a);
    unpack8<T>(x, b);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s = fmaf(a[i], b[i], s);
    return s;
}

// ---------------------------------------------------------------------------
// 2: head logits l_k = Wa2[k] . h + ba2_k, selection l_k > 0; Y[t] = y.  One CTA per head:
// its logit and decision, and for a selected head the positions p < t with no K/V row yet
// (ascending, by head).  The CTA that finishes last writes the ascending head list, its
// length and the q/k/v kernel's work-unit prefix (atomic ticket, reset for the next step).
constexpr int kSelThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kSelThreads) k_attn_select(const AParams p)
{
    __shared__ float red[kSelThreads / 32];
    __shared__ int wcnt[kSelThreads / 32];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, k = blockIdx.x;
    const int t = *p.tcur;
    const bool full = t >= p.tmax;
    if (k == 0 && !full) {
        const uint4* src = reinterpret_cast<const uint4*>(p.y);
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.Y) + (size_t)t * p.d);
        for (int v = tid; v < p.d / 8; v += kSelThreads) dst[v] = src[v];
    }
    const int hv = p.Ha / 8;
    const uint4* w = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.Wa2) + (size_t)k * p.Ha);
    float acc = 0.f;
    for (int v = tid; v < hv; v += kSelThreads) {
        float wf[8];
        unpack8<T>(ldg_stream(w + v), wf);
        const float4 a = reinterpret_cast<const float4*>(p.h)[2 * v], b = reinterpret_cast<const float4*>(p.h)[2 * v + 1];
        acc = fmaf(wf[0], a.x, acc); acc = fmaf(wf[1], a.y, acc); acc = fmaf(wf[2], a.z, acc); acc = fmaf(wf[3], a.w, acc);
        acc = fmaf(wf[4], b.x, acc); acc = fmaf(wf[5], b.y, acc); acc = fmaf(wf[6], b.z, acc); acc = fmaf(wf[7], b.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
    const float bias = p.ba2 ? DT<T>::f(reinterpret_cast<const T*>(p.ba2)[k]) : 0.f;
    const bool on = !full && ((red[0] + red[1]) + (red[2] + red[3])) + bias > 0.f;
    if (on) {
        // missing K/V rows of this head, ascending: an ordered block-wide compaction
        const uint8_t* f = p.filled + (size_t)k * p.tmax;
        uint16_t* ml = p.miss + (size_t)k * p.tmax;
        int m = 0;
        for (int p0 = 0; p0 < t; p0 += kSelThreads) {
            const bool miss = p0 + tid < t && !f[p0 + tid];
            const uint32_t bal = __ballot_sync(0xffffffffu, miss);
            if (lane == 0) wcnt[warp] = __popc(bal);
            __syncthreads();
            int base = m;
            for (int q = 0; q < warp; ++q) base += wcnt[q];
            if (miss) ml[base + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)(p0 + tid);
            m += (wcnt[0] + wcnt[1]) + (wcnt[2] + wcnt[3]);
            __syncthreads();
        }
        if (tid == 0) p.nmiss[k] = m;
    }
    if (tid == 0) p.hsel[k] = on ? 1 : 0;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(p.sticket, 1u) == (uint32_t)(gridDim.x - 1);
    __syncthreads();
    if (!s_last || warp != 0) return;
    __threadfence();
    // ascending head list and the q/k/v work units per head slot (its q rows in groups of kRW,
    // then the k and v row groups once per group of kPos positions: the new token and the
    // missing ones), with their exclusive prefix
    int m = 0, run = 0;
    for (int k0 = 0; k0 < p.nh; k0 += 32) {
        const int kk = k0 + lane;
        const bool o = kk < p.nh && __ldcg(p.hsel + kk) != 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, o);
        const int u = o ? (p.dh / kRW) * (1 + 2 * ((__ldcg(p.nmiss + kk) + kPos) / kPos)) : 0;
        int x = u;
#pragma unroll
        for (int q = 1; q < 32; q <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, q);
            if (lane >= q) x += y;
        }
        if (o) {
            const int slot = m + __popc(bal & ((1u << lane) - 1u));
            p.heads[slot] = kk;
            p.upref[slot] = run + x - u;
        }
        run += __shfl_sync(0xffffffffu, x, 31);
        m += __popc(bal);
    }
    if (lane == 0) {
        *p.count = m;
        p.upref[m] = run;
        *p.sticket = 0u;                                // ready for the next step
        if (full) latch(p.err, ERR_CACHE_FULL);
    }
}

// ---------------------------------------------------------------------------
// 3: q, k, v rows of the selected heads for the new token; missing K/V rows from Y[p].
// Work units, balanced over every warp of the grid (warp w takes the w-th of W equal
// contiguous ranges): per head slot, its q rows in pairs (the new token), then for each pair
// of k rows and of v rows one unit per group of kPos positions (the new token first, then
// the missing positions in order).  Contiguous ranges keep a CTA's warps on one head, so the
// few stored input rows Y[p] they all read stay in L1, and the units of one weight-row pair
// run back to back on one warp.  The new token was stored in Y by the select kernel.

// each position accumulates lane-strided in ascending vector order, then a warp sum.
// Dot products of two weight rows w0, w1 with NP input rows y_j over a d-length row: each
// 16-byte input vector is loaded once for both weight rows (the input rows are the traffic
// that repeats across a head's weight rows).  U vector columns per lane in flight; each sum
// accumulates lane-strided in ascending vector order, then a warp sum.
template <typename T, int R, int NP, int U>
__device__ __forceinline__ void rows_dotR(const uint4* const* w, const uint4* const* y, int nv, int lane, float (*z)[kPos]) {
    float a[R][NP];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < NP; ++j) a[r][j] = 0.f;
    int v = lane;
    for (; v + 32 * (U - 1) < nv; v += 32 * U) {
        uint4 wv[U][R], yv[U][NP];
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int r = 0; r < R; ++r) wv[u][r] = __ldg(w[r] + v + 32 * u);
#pragma unroll
            for (int j = 0; j < NP; ++j) yv[u][j] = __ldg(y[j] + v + 32 * u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int j = 0; j < NP; ++j) a[r][j] += dot8<T>(wv[u][r], yv[u][j]);
    }
    for (; v < nv; v += 32) {
        uint4 wv[R];
#pragma unroll
        for (int r = 0; r < R; ++r) wv[r] = __ldg(w[r] + v);
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            const uint4 yv = __ldg(y[j] + v);
#pragma unroll
            for (int r = 0; r < R; ++r) a[r][j] += dot8<T>(wv[r], yv);
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < NP; ++j) z[r][j] = warp_sum(a[r][j]);
}

template <typename T>
__global__ void __launch_bounds__(256) k_attn_qkv(const AParams p)
{
    __shared__ int up[1025];
    const int lane = threadIdx.x & 31;
    const int t = *p.tcur, count = *p.count;
    if (t >= p.tmax || count == 0) return;
    for (int s = threadIdx.x; s <= count; s += 256) up[s] = p.upref[s];
    __syncthreads();
    const int nv = p.d / 8, dh = p.dh, hp = dh / kRW, total = up[count], W = gridDim.x * 8;
    const T* Yh = reinterpret_cast<const T*>(p.Y);
    const uint4* yt = reinterpret_cast<const uint4*>(Yh + (size_t)t * p.d);
    const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int u0 = (int)((long long)total * gw / W), u1 = (int)((long long)total * (gw + 1) / W);
    for (int u = u0; u < u1; ++u) {
        int lo = 0, hi = count - 1;                     // the slot: last s with up[s] <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (up[mid] <= u) lo = mid; else hi = mid - 1;
        }
        const int s = lo, h = p.heads[s];
        int w = u - up[s];
        if (w < hp) {                                   // q rows 2w, 2w + 1 for the new token
            const int i = kRW * w;
            const size_t row = (size_t)h * dh + i;
            const T* Wq = reinterpret_cast<const T*>(p.Wq);
            const uint4* wr[kRW];
#pragma unroll
            for (int r = 0; r < kRW; ++r) wr[r] = reinterpret_cast<const uint4*>(Wq + (row + r) * p.d);
            float z[kRW][kPos];
            rows_dotR<T, kRW, 1, 2>(wr, &yt, nv, lane, z);
            if (lane == 0) {
                const T* bq = reinterpret_cast<const T*>(p.bq);
#pragma unroll
                for (int r = 0; r < kRW; ++r) p.q[(size_t)s * dh + i + r] = z[r][0] + (bq ? DT<T>::f(bq[row + r]) : 0.f);
            }
            continue;
        }
        w -= hp;
        const int nm = p.nmiss[h], ng = (nm + kPos) / kPos;
        const int type = w / (hp * ng);                 // 0: k rows, 1: v rows
        const int rem = w - type * hp * ng, ip = rem / ng, g = rem - ip * ng;
        const int i = kRW * ip;
        const size_t row = (size_t)h * dh + i;
        const T* Wr = reinterpret_cast<const T*>(type == 0 ? p.Wk : p.Wv);
        const T* br = reinterpret_cast<const T*>(type == 0 ? p.bk : p.bv);
        const uint4* wr[kRW];
#pragma unroll
        for (int r = 0; r < kRW; ++r) wr[r] = reinterpret_cast<const uint4*>(Wr + (row + r) * p.d);
        const uint16_t* ml = p.miss + (size_t)h * p.tmax;
        const int j0 = g * kPos, np = min(kPos, nm + 1 - j0);
        int pos[kPos];
        const uint4* yr[kPos];
#pragma unroll
        for (int j = 0; j < kPos; ++j) {
            const int jj = j0 + min(j, np - 1);
            pos[j] = jj == 0 ? t : (int)ml[jj - 1];
            yr[j] = reinterpret_cast<const uint4*>(Yh + (size_t)pos[j] * p.d);
        }
        float z[kRW][kPos];
        switch (np) {
            case 1: rows_dotR<T, kRW, 1, 2>(wr, yr, nv, lane, z); break;
            case 2: rows_dotR<T, kRW, 2, 1>(wr, yr, nv, lane, z); break;
            case 3: rows_dotR<T, kRW, 3, 1>(wr, yr, nv, lane, z); break;
            default: rows_dotR<T, kRW, 4, 1>(wr, yr, nv, lane, z); break;
        }
        if (lane == 0) {
            T* C = reinterpret_cast<T*>(type == 0 ? p.K : p.V);
#pragma unroll
            for (int j = 0; j < kPos; ++j)
                if (j < np) {
                    T* dst = C + ((size_t)h * p.tmax + pos[j]) * dh + i;
#pragma unroll
                    for (int r = 0; r < kRW; ++r) dst[r] = DT<T>::r(z[r][j] + (br ? DT<T>::f(br[row + r]) : 0.f));
                }
        }
    }
}

// ---------------------------------------------------------------------------
// 4: o_k = softmax(q . K / sqrt(dh)) V over positions 0..t for every selected head.
// Items (head slot, split of the positions); each warp walks its positions in order
// with an online softmax (running max, sum and weighted V); the CTA's warps and then
// the head's splits are combined in fixed order.  Marks the rows used as filled.
template <typename T>
__global__ void __launch_bounds__(256, 1) k_attn_core(const AParams p)
{
    __shared__ float qs[256];
    __shared__ float wm[8], wz[8];
    __shared__ float wo[8][256];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = *p.tcur, count = *p.count;
    if (t >= p.tmax || count == 0) return;
    const int T_ = t + 1, dh = p.dh, Sa = p.Sa;
    const int E = (dh + 31) / 32;                      // elements per lane (dh <= 256: E <= 8)
    const float scale = 1.0f / sqrtf((float)dh);
    const T* Kc = reinterpret_cast<const T*>(p.K);
    const T* Vc = reinterpret_cast<const T*>(p.V);
    for (int it = blockIdx.x; it < count * Sa; it += gridDim.x) {
        const int s = it / Sa, sp = it % Sa, h = p.heads[s];
        const int p0 = (int)((long long)T_ * sp / Sa), p1 = (int)((long long)T_ * (sp + 1) / Sa);
        __syncthreads();
        for (int e = tid; e < dh; e += 256) qs[e] = p.q[(size_t)s * dh + e];
        __syncthreads();
        float m = -INFINITY, z = 0.f, o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = 0.f;
        // this warp's share of the split's positions, 32 at a time: lane i scores position
        // base + i (its whole K row in 16-byte loads, issued together), the chunk's running
        // max and sum follow, then each lane adds p_i V[base + i] over its E elements of the
        // output, positions in order (eight rows' loads in flight at a time)
        const int w0 = p0 + (int)((long long)(p1 - p0) * warp / 8), w1 = p0 + (int)((long long)(p1 - p0) * (warp + 1) / 8);
        const int nvk = dh / 8;
        const T* Kh = Kc + (size_t)h * p.tmax * dh;
        const T* Vh = Vc + (size_t)h * p.tmax * dh;
        for (int base = w0; base < w1; base += 32) {
            const int n = min(32, w1 - base);
            float sc = -INFINITY;
            if (lane < n) {
                const uint4* kr = reinterpret_cast<const uint4*>(Kh + (size_t)(base + lane) * dh);
                float a0 = 0.f, a1 = 0.f;
                auto qdot = [&](const uint4& kv4, int v) {
                    float kf[8];
                    unpack8<T>(kv4, kf);
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) a = fmaf(qs[8 * v + e], kf[e], a);
                    return a;
                };
                int v = 0;
                for (; v + 3 < nvk; v += 4) {
                    const uint4 k0 = __ldcg(kr + v), k1 = __ldcg(kr + v + 1), k2 = __ldcg(kr + v + 2), k3 = __ldcg(kr + v + 3);
                    a0 += qdot(k0, v); a1 += qdot(k1, v + 1); a0 += qdot(k2, v + 2); a1 += qdot(k3, v + 3);
                }
                for (; v < nvk; ++v) a0 += qdot(__ldcg(kr + v), v);
                sc = (a0 + a1) * scale;
            }
            float mc = sc;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, off));
            const float mn = fmaxf(m, mc);
            const float cf = expf(m - mn);
            const float ev = lane < n ? expf(sc - mn) : 0.f;
            z = z * cf + warp_sum(ev);
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] *= cf;
            for (int i0 = 0; i0 < n; i0 += 8) {
                float vv[8][8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const T* vr = Vh + (size_t)(base + i0 + (i0 + j < n ? j : 0)) * dh;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int c = lane * E + e;
                        vv[j][e] = (e < E && c < dh) ? DT<T>::f(__ldcg(vr + c)) : 0.f;
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (i0 + j < n) {
                        const float pj = __shfl_sync(0xffffffffu, ev, i0 + j);
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[e] = fmaf(pj, vv[j][e], o[e]);
                    }
                }
            }
            m = mn;
        }
        if (lane == 0) { wm[warp] = m; wz[warp] = z; }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int c = lane * E + e;
            if (e < E && c < dh) wo[warp][c] = o[e];
        }
        for (int pos = p0 + tid; pos < p1; pos += 256) p.filled[(size_t)h * p.tmax + pos] = 1;
        __syncthreads();
        // this split: combine the warps in order
        float* part = p.opart + ((size_t)s * Sa + sp) * (dh + 2);
        if (tid == 0) {
            float M = -INFINITY;
            for (int w = 0; w < 8; ++w) if (wz[w] > 0.f) M = fmaxf(M, wm[w]);
            float Z = 0.f;
            for (int w = 0; w < 8; ++w) if (wz[w] > 0.f) Z += wz[w] * expf(wm[w] - M);
            part[0] = M;
            part[1] = Z;
        }
        for (int c = tid; c < dh; c += 256) {
            float M = -INFINITY;
            for (int w = 0; w < 8; ++w) if (wz[w] > 0.f) M = fmaxf(M, wm[w]);
            float O = 0.f;
            for (int w = 0; w < 8; ++w) if (wz[w] > 0.f) O += wo[w][c] * expf(wm[w] - M);
            part[2 + c] = O;
        }
        // the head's last split to finish combines all splits in order
        __threadfence();
        __syncthreads();
        if (tid == 0) s_last = atomicAdd(&p.tickets[s], 1u) == (uint32_t)(Sa - 1);
        __syncthreads();
        if (s_last) {
            __threadfence();
            const float* pa = p.opart + (size_t)s * Sa * (dh + 2);
            float M = -INFINITY;
            for (int q = 0; q < Sa; ++q) {
                const float zq = __ldcg(pa + (size_t)q * (dh + 2) + 1);
                if (zq > 0.f) M = fmaxf(M, __ldcg(pa + (size_t)q * (dh + 2)));
            }
            float Z = 0.f;
            for (int q = 0; q < Sa; ++q) {
                const float zq = __ldcg(pa + (size_t)q * (dh + 2) + 1);
                if (zq > 0.f) Z += zq * expf(__ldcg(pa + (size_t)q * (dh + 2)) - M);
            }
            for (int c = tid; c < dh; c += 256) {
                float O = 0.f;
                for (int q = 0; q < Sa; ++q) {
                    const float zq = __ldcg(pa + (size_t)q * (dh + 2) + 1);
                    if (zq > 0.f) O += __ldcg(pa + (size_t)q * (dh + 2) + 2 + c) * expf(__ldcg(pa + (size_t)q * (dh + 2)) - M);
                }
                p.o[(size_t)s * dh + c] = O / Z;
            }
            if (tid == 0) p.tickets[s] = 0u;
        }
    }
}

// ---------------------------------------------------------------------------
// 5: out = bo + sum over the R = count dh selected rows of o_k[i] WoT[k dh + i]
// (WoT head-major: each row contiguous).  CTA c owns the 8-column vectors
// [8c, 8c + 8) of out, so no partials leave the CTA: thread (row lane rl, vector
// j) walks rows rl, rl + 64, ... eight at a time (eight loads in flight), then the
// 64 row lanes are added in a fixed order.  The last step: the position advances
// (no CTA of this kernel reads it; a full cache already gave count = 0).
constexpr int kOutVec = 8, kOutLanes = 64;

template <typename T>
__global__ void __launch_bounds__(kOutVec * kOutLanes) k_attn_out(const AParams p)
{
    __shared__ float red[kOutLanes][kOutVec][8];
    const int tid = threadIdx.x, j = tid % kOutVec, rl = tid / kOutVec;
    const int nv = p.d / 8, v = blockIdx.x * kOutVec + j, dh = p.dh;
    const int R = *p.count * dh;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const T* Wo = reinterpret_cast<const T*>(p.WoT);
    auto row_ptr = [&](int r) {
        const int s = r / dh;
        return reinterpret_cast<const uint4*>(Wo + ((size_t)p.heads[s] * dh + (r - s * dh)) * p.d) + v;
    };
    auto fold = [&](const uint4& w, float a) {
        float wf[8];
        unpack8<T>(w, wf);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(a, wf[e], acc[e]);
    };
    if (v < nv) {
        int r = rl;
        for (; r + 7 * kOutLanes < R; r += 8 * kOutLanes) {
            uint4 w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = ldg_stream(row_ptr(r + k * kOutLanes));
#pragma unroll
            for (int k = 0; k < 8; ++k) fold(w[k], __ldcg(p.o + r + k * kOutLanes));
        }
        for (; r < R; r += kOutLanes) fold(ldg_stream(row_ptr(r)), __ldcg(p.o + r));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rl][j][e] = acc[e];
    __syncthreads();
    if (tid < kOutVec * 8) {
        const int jj = tid / 8, e = tid % 8, vv = blockIdx.x * kOutVec + jj;
        if (vv < nv) {
            float sum = 0.f;
            for (int q = 0; q < kOutLanes; ++q) sum += red[q][jj][e];
            const int col = vv * 8 + e;
            p.out[col] = sum + (p.bo ? DT<T>::f(reinterpret_cast<const T*>(p.bo)[col]) : 0.f);
        }
    }
    if (blockIdx.x == 0 && tid == 0) {
        const int t = *p.tcur;
        if (t < p.tmax) *p.tcur = t + 1;
    }
}

bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

bool valid(const spffn_attn_config* c) {
    if (!c) return false;
    if (c->d < 64 || c->d > 16384 || c->d % 64) return false;
    if (c->nh < 1 || c->nh > 1024) return false;
    if (c->dh < 8 || c->dh > 256 || c->dh % 8) return false;
    if (c->Ha < 64 || c->Ha > 8192 || c->Ha % 64) return false;
    if (c->tmax < 1 || c->tmax > 16384) return false;
    if (c->dtype != SPFFN_F16 && c->dtype != SPFFN_BF16) return false;
    return c->flags == 0;
}

int sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n <= 0) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

}  // namespace
}  // namespace spffn

struct spffn_attn_ctx {
    spffn_attn_config cfg;
    spffn_attn_weights w;
    char* ws;
    spffn::ALayout lay;
    int qkv_blocks;                                     // resident CTAs of the q/k/v kernel
};

using namespace spffn;

namespace {

AParams attn_params(const spffn_attn_ctx& c, const void* y, int32_t* heads, int32_t* count, float* out) {
    AParams p;
    memset(&p, 0, sizeof(p));
    const auto& w = c.w;
    p.Wq = w.Wq; p.bq = w.bq; p.Wk = w.Wk; p.bk = w.bk; p.Wv = w.Wv; p.bv = w.bv; p.WoT = w.WoT; p.bo = w.bo;
    p.Wa2 = w.Wa2; p.ba2 = w.ba2;
    p.y = y;
    p.d = c.cfg.d; p.nh = c.cfg.nh; p.dh = c.cfg.dh; p.Ha = c.cfg.Ha; p.tmax = c.cfg.tmax; p.Sa = c.lay.Sa;
    uint32_t* ctl = reinterpret_cast<uint32_t*>(c.ws + c.lay.ctl);
    p.err = ctl;
    p.tcur = reinterpret_cast<int32_t*>(ctl + 1);
    p.heads = heads;
    p.count = count;
    p.h = reinterpret_cast<const float*>(c.ws + c.lay.h);
    p.q = reinterpret_cast<float*>(c.ws + c.lay.q);
    p.miss = reinterpret_cast<uint16_t*>(c.ws + c.lay.miss);
    p.nmiss = reinterpret_cast<int32_t*>(c.ws + c.lay.nmiss);
    p.hsel = reinterpret_cast<int32_t*>(c.ws + c.lay.hsel);
    p.sticket = ctl + 2;
    p.upref = reinterpret_cast<int32_t*>(c.ws + c.lay.upref);
    p.opart = reinterpret_cast<float*>(c.ws + c.lay.opart);
    p.o = reinterpret_cast<float*>(c.ws + c.lay.o);
    p.tickets = reinterpret_cast<uint32_t*>(c.ws + c.lay.tickets);
    p.K = c.ws + c.lay.K;
    p.V = c.ws + c.lay.V;
    p.filled = reinterpret_cast<uint8_t*>(c.ws + c.lay.filled);
    p.Y = c.ws + c.lay.Y;
    p.out = out;
    return p;
}

template <typename T>
cudaError_t step_impl(const spffn_attn_ctx& c, const AParams& p, cudaStream_t st) {
    const int G = c.lay.S;
    cudaError_t e = launch_hidden(c.cfg.dtype, c.w.Wa1, c.w.ba1, p.y, 1, c.cfg.d, c.cfg.Ha,
                                  reinterpret_cast<float*>(c.ws + c.lay.h), G, st);
    if (e != cudaSuccess) return e;
    k_attn_select<T><<<c.cfg.nh, kSelThreads, 0, st>>>(p);
    k_attn_qkv<T><<<c.qkv_blocks, 256, 0, st>>>(p);   // every resident warp takes units
    k_attn_core<T><<<G, 256, 0, st>>>(p);
    k_attn_out<T><<<(c.cfg.d / 8 + kOutVec - 1) / kOutVec, kOutVec * kOutLanes, 0, st>>>(p);
    return cudaGetLastError();
}

spffn_status status_of(cudaError_t e) { return e == cudaSuccess ? SPFFN_OK : SPFFN_ERR_CUDA; }

}  // namespace

extern "C" {

size_t spffn_attn_workspace_bytes(const spffn_attn_config* cfg) {
    if (!valid(cfg)) return 0;
    return attn_layout(*cfg, sms()).total;
}

spffn_status spffn_attn_create(const spffn_attn_config* cfg, const spffn_attn_weights* w, void* workspace,
                               size_t workspace_bytes, spffn_attn_ctx** out) {
    if (!out) return SPFFN_ERR_INVALID_ARG;
    *out = nullptr;
    if (!valid(cfg) || !w || !w->Wq || !w->Wk || !w->Wv || !w->WoT || !w->Wa1 || !w->Wa2) return SPFFN_ERR_INVALID_ARG;
    const void* all[] = {w->Wq, w->bq, w->Wk, w->bk, w->Wv, w->bv, w->WoT, w->bo, w->Wa1, w->ba1, w->Wa2, w->ba2};
    for (const void* q : all)
        if (q && !aligned16(q)) return SPFFN_ERR_INVALID_ARG;
    const ALayout lay = attn_layout(*cfg, sms());
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SPFFN_ERR_WORKSPACE;
    if (workspace_bytes < lay.total) return SPFFN_ERR_WORKSPACE;
    spffn_attn_ctx* c = new (std::nothrow) spffn_attn_ctx();
    if (!c) return SPFFN_ERR_UNSUPPORTED;
    c->cfg = *cfg;
    c->w = *w;
    c->ws = static_cast<char*>(workspace);
    c->lay = lay;
    int occ = 0;
    const cudaError_t e = cfg->dtype == SPFFN_BF16
                              ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_attn_qkv<__nv_bfloat16>, 256, 0)
                              : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_attn_qkv<__half>, 256, 0);
    if (e != cudaSuccess || occ < 1) {
        cudaGetLastError();
        occ = 2;
    }
    c->qkv_blocks = lay.S * std::min(occ, 8);
    *out = c;
    return SPFFN_OK;
}

spffn_status spffn_attn_destroy(spffn_attn_ctx* ctx) {
    delete ctx;
    return SPFFN_OK;
}

spffn_status spffn_attn_reset(spffn_attn_ctx* ctx, void* stream) {
    if (!ctx) return SPFFN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ctx->ws + ctx->lay.ctl + 4, 0, 4, st);                  // t = 0
    if (e == cudaSuccess)
        e = cudaMemsetAsync(ctx->ws + ctx->lay.filled, 0, (size_t)ctx->cfg.nh * ctx->cfg.tmax, st);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(ctx->ws + ctx->lay.tickets, 0, (size_t)ctx->cfg.nh * sizeof(uint32_t), st);
    return status_of(e);
}

spffn_status spffn_attn_step(spffn_attn_ctx* ctx, const void* y, int32_t* heads, int32_t* count, float* out,
                             void* stream) {
    if (!ctx || !y || !heads || !count || !out) return SPFFN_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out)) return SPFFN_ERR_INVALID_ARG;
    const AParams p = attn_params(*ctx, y, heads, count, out);
    cudaStream_t st = (cudaStream_t)stream;
    return status_of(ctx->cfg.dtype == SPFFN_BF16 ? step_impl<__nv_bfloat16>(*ctx, p, st)
                                                  : step_impl<__half>(*ctx, p, st));
}

spffn_status spffn_attn_cache(spffn_attn_ctx* ctx, spffn_attn_cache_view* view) {
    if (!ctx || !view) return SPFFN_ERR_INVALID_ARG;
    view->K = ctx->ws + ctx->lay.K;
    view->V = ctx->ws + ctx->lay.V;
    view->filled = reinterpret_cast<const uint8_t*>(ctx->ws + ctx->lay.filled);
    view->Y = ctx->ws + ctx->lay.Y;
    view->t = reinterpret_cast<const int32_t*>(ctx->ws + ctx->lay.ctl + 4);
    return SPFFN_OK;
}

int32_t spffn_attn_step_kernel_launches(void) { return 5; }

spffn_status spffn_attn_last_device_error(spffn_attn_ctx* ctx, uint32_t* code, void* stream) {
    if (!ctx) return SPFFN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    uint32_t* err = reinterpret_cast<uint32_t*>(ctx->ws + ctx->lay.ctl);
    if (cudaMemcpyAsync(&v, err, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SPFFN_ERR_CUDA;
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess) return SPFFN_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SPFFN_ERR_CUDA;
    if (code) *code = v;
    return v ? SPFFN_ERR_DEVICE_CHECK : SPFFN_OK;
}

}  // extern "C"
