// Persistent whole-stack decode kernel for small batches (B <= 2).
//
// One CTA per SM runs every layer of the stack in a single launch.  CTA c owns
// a contiguous span of Wp1 rows (predictor hidden units), a contiguous span of
// Wp2 rows (FFN neurons, placed hot-first and dealt over the spans offline) and
// a slice of the output columns.  Per layer l:
//   A  x_l from the previous layer's u; h = ReLU(Wp1 x + bp1) on own Wp1 rows
//      -- grid barrier --
//   B  logits of own neurons, threshold (union over the batch) and the CTA's
//      ascending list of selected neurons; the FFN of exactly those neurons:
//      FC1 vec_dot + bias + ReLU, FC2 AXPY into a per-CTA fp32 partial
//      -- grid barrier --
//   D  y = b2 + the G partials in fixed order on own columns, u = x + y; the
//      neuron table (each CTA's list at its prefix position) and its count
//      -- grid barrier --
// With look-ahead prediction (DejaVu's asynchronous predictor) the set of layer
// l+1 is predicted from x_l: h_{l+1} and FFN_l share one phase, logits_{l+1}
// and the reduction of y_l the next, so a layer has two grid barriers.
//
// Weight bytes move with cp.async.bulk (TMA bulk copies) into shared-memory
// rings guarded by mbarriers.  The predictor weights do not depend on the
// data, so a dedicated producer warp streams them ahead across the grid
// barriers (the ring keeps HBM busy while the consumers wait); a second
// producer warp gathers the FFN rows as soon as the neuron table is known.
//
// Every wait is bounded (globaltimer): on expiry the CTA latches an error,
// raises a grid-wide abort flag, stops issuing copies, waits (bounded) for the
// copies it already issued and returns.
#include <cstring>
#include "spffn_fused.cuh"

namespace spffn {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 64;      // + predictor producer warp + FFN producer warp
constexpr int kMaxFusedLayers = 128;
constexpr int kMaxVPT = 5;                      // 16-byte column vectors per consumer thread (d <= 10240)
constexpr int kMaxG = 256;
constexpr unsigned long long kWaitNs = 2000000000ull;   // 2 s per wait (grid barriers: p.wait_ns)
constexpr int kTraceMarks = 16;                 // stamps per (CTA, layer), see TRACE() below
constexpr int kMaxMaskWords = 2048;             // n <= 65536 on this path

struct LayerW {
    const void *W1, *b1, *W2T, *b2, *Wp1, *bp1, *Wp2, *bp2;
    int32_t* idx;
    const int32_t* tab;        // caller-tables mode: this layer's neuron table and its length (device)
    const int32_t* tab_count;
};

struct Params {
    int L, B, d, n, H, G;
    const void* x_in;
    void* x_out;
    float* y;
    int32_t* counts;
    uint32_t* bar;        // grid-barrier counter
    uint32_t* err;
    uint32_t* abort;
    int32_t* cta_count;   // [2][G + 1] list lengths per CTA, by list parity
    float* h;             // [2][NB][H]: h of predictor layer q in buffer q & 1
    float* partial;       // [G][B][d]
    float* u;             // [B][d]
    int pred_slots, pred_slot_bytes, ffn_slots, R1, R2, max_rows;
    unsigned long long wait_ns;  // limit of a grid-barrier wait (other waits: kWaitNs)
    uint32_t bar_extra;          // arrivals a grid barrier expects beyond G (0; 1 only under the wait test)
    int hot_rows;                // > 0: the first hot_rows slots of every dealt range stay in L2 (evict_last)
                                 // and the predictor and the other FFN rows are copied evict_first
    unsigned long long* trace;   // optional [G][L][kTraceMarks] globaltimer stamps
    LayerW layer[kMaxFusedLayers];
};

// ---------------------------------------------------------------------------
// PTX wrappers
__device__ __forceinline__ uint32_t sptr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long gtime() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sptr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sptr(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sptr(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(sptr(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(sptr(dst)),
        "l"(src), "r"(bytes), "r"(sptr(bar))
        : "memory");
}
// the same with an L2 eviction-priority policy for the copied lines (createpolicy)
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(sptr(dst)), "l"(src), "r"(bytes), "r"(sptr(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// offset of neuron slot j inside its dealt range (ranges c = [floor(n c / G), floor(n (c+1) / G)));
// after the hot-first dealt placement, offset k holds the (k G + c)-th hottest neuron
__device__ __forceinline__ int range_offset(int j, int n, int G) {
    int c = (int)((long long)j * G / n);
    while (c + 1 < G && (int)((long long)n * (c + 1) / G) <= j) ++c;
    while (c > 0 && (int)((long long)n * c / G) > j) --c;
    return j - (int)((long long)n * c / G);
}
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

struct Shared {
    uint64_t* pfull;
    uint64_t* pempty;
    uint64_t* ffull;
    uint64_t* fempty;
    volatile int* flags;     // [0] local abort, [1] list tag|length, [2] pred issued, [3] ffn issued,
                             // [4] pred done, [5] ffn done, [7] last final list + 1
    char* pring;
    char* fring;
    void* xs;
    float* hs;
    unsigned char* sel;
    int32_t* nl;             // [2][max_rows] neuron lists, by list parity
    float* bias1;            // [max_rows_h] bp1 for the CTA's Wp1 rows
    float* bias2;            // [max_rows]   bp2 for the CTA's Wp2 rows
    float* biasy;            // [max_cols]   b2 for the CTA's output columns
    float* red;              // FC1 partial dots: [2][4][8] for neuron quads (B = 1), then
                             // [2][8][2][NB] for pairs, each by step parity
    float* red2;             // [8][NB]
    float* red1;             // [32][8][NB] GEMV1 row partials per warp
    float* misc;             // [16]
};

__device__ __forceinline__ bool aborted(const Shared& S, const Params& p) {
    return S.flags[0] != 0 || *(volatile uint32_t*)p.abort != 0;
}

__device__ __forceinline__ void raise_abort(const Shared& S, const Params& p, uint32_t bits) {
    S.flags[0] = 1;
    atomicOr(p.err, bits);
    atomicExch(p.abort, 1u);
}

// Bounded wait on an mbarrier phase; false on timeout (or abort, for a producer).
// Consumer threads ignore the abort flag here: a phase either completes for all
// of them or for none, so every consumer leaves a wait the same way and no
// named barrier is left short of arrivals.
__device__ __forceinline__ bool wait_bounded(const Shared& S, const Params& p, uint64_t* b, uint32_t parity,
                             bool producer = false) {
    if (mbar_try(b, parity)) return true;
    const unsigned long long t0 = gtime();
    while (!mbar_try(b, parity)) {
        if (producer && aborted(S, p)) return false;
        if (gtime() - t0 > kWaitNs) {
            raise_abort(S, p, ERR_PIPE_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Grid barrier among the consumer groups of all CTAs (monotonic counter).
__device__ __forceinline__ bool grid_barrier(const Shared& S, const Params& p, uint32_t& epoch) {
    consumer_sync();
    epoch += 1;
    if (threadIdx.x == 0) {
        // the CTA barrier above orders every consumer's writes before this release
        red_release_add(p.bar, 1u);
        const uint32_t target = epoch * ((uint32_t)p.G + p.bar_extra);
        if (ld_acquire(p.bar) < target) {
            const unsigned long long t0 = gtime();
            while (ld_acquire(p.bar) < target) {
                if (*(volatile uint32_t*)p.abort) { S.flags[0] = 1; break; }
                if (gtime() - t0 > p.wait_ns) { raise_abort(S, p, ERR_BARRIER_TIMEOUT); break; }
            }
        }
    }
    consumer_sync();
    return S.flags[0] == 0;
}

__device__ __forceinline__ int split_lo(int total, int parts, int i) {
    return (int)((long long)total * i / parts);
}

// ---------------------------------------------------------------------------
// arithmetic helpers
//
// Weight x activation products where both are in the storage dtype (GEMV1 and
// FC1) use the mixed-precision FMA of sm_100 (fp16/bf16 operands, fp32
// accumulator: the product is exact, one rounding).  Products with fp32
// activations (GEMV2 with h, FC2 with a) convert the weight pair and use the
// packed two-lane fp32 FMA.
typedef unsigned long long u64;

constexpr uint32_t kWaitHintNs = 1000000;        // suspend-time hint of a consumer's mbarrier wait

__device__ __forceinline__ u64 pk(float a, float b) {
    u64 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 upk(u64 r) {
    float2 f;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(r));
    return f;
}
__device__ __forceinline__ void ffma2(u64& acc, u64 a, u64 b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

template <typename T> struct Arith;
template <> struct Arith<__half> {
    // a0 += w.lo * x.lo ; a1 += w.hi * x.hi  (w, x: packed pairs of fp16)
    static __device__ __forceinline__ void mix2(float& a0, float& a1, uint32_t w, uint32_t x) {
        unsigned short wl, wh, xl, xh;
        asm("mov.b32 {%0, %1}, %2;" : "=h"(wl), "=h"(wh) : "r"(w));
        asm("mov.b32 {%0, %1}, %2;" : "=h"(xl), "=h"(xh) : "r"(x));
        asm("fma.rn.f32.f16 %0, %1, %2, %0;" : "+f"(a0) : "h"(wl), "h"(xl));
        asm("fma.rn.f32.f16 %0, %1, %2, %0;" : "+f"(a1) : "h"(wh), "h"(xh));
    }
    static __device__ __forceinline__ u64 widen2(uint32_t w) {
        const float2 f = DT<__half>::f2(w);
        return pk(f.x, f.y);
    }
};
template <> struct Arith<__nv_bfloat16> {
    static __device__ __forceinline__ void mix2(float& a0, float& a1, uint32_t w, uint32_t x) {
        unsigned short wl, wh, xl, xh;
        asm("mov.b32 {%0, %1}, %2;" : "=h"(wl), "=h"(wh) : "r"(w));
        asm("mov.b32 {%0, %1}, %2;" : "=h"(xl), "=h"(xh) : "r"(x));
        asm("fma.rn.f32.bf16 %0, %1, %2, %0;" : "+f"(a0) : "h"(wl), "h"(xl));
        asm("fma.rn.f32.bf16 %0, %1, %2, %0;" : "+f"(a1) : "h"(wh), "h"(xh));
    }
    static __device__ __forceinline__ u64 widen2(uint32_t w) {
        return pk(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
};

// 16-byte weight vector . 16-byte storage-dtype vector into four partial sums
template <typename T>
__device__ __forceinline__ void dot_mix(float* a, const uint4& w, const uint4& x) {
    Arith<T>::mix2(a[0], a[1], w.x, x.x);
    Arith<T>::mix2(a[2], a[3], w.y, x.y);
    Arith<T>::mix2(a[0], a[1], w.z, x.z);
    Arith<T>::mix2(a[2], a[3], w.w, x.w);
}

__device__ __forceinline__ float sum4(const float* a) { return (a[0] + a[1]) + (a[2] + a[3]); }

__device__ __forceinline__ bool mbar_try_hint(uint64_t* b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(sptr(b)), "r"(parity), "r"(kWaitHintNs)
        : "memory");
    return ok != 0;
}

// Consumer-side bounded wait: suspends in hardware between checks.
__device__ __forceinline__ bool cwait(const Shared& S, const Params& p, uint64_t* b, uint32_t parity) {
    if (mbar_try(b, parity)) return true;
    const unsigned long long t0 = gtime();
    while (!mbar_try_hint(b, parity)) {
        if (gtime() - t0 > kWaitNs) {
            raise_abort(S, p, ERR_PIPE_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Phase stamps (only when a trace buffer is bound): consumer thread 0 records
// %globaltimer at fixed points of each layer.
#define TRACE(mark)                                                                                  \
    do {                                                                                             \
        if (p.trace && tid == 0 && l < p.L)                                                          \
            p.trace[((size_t)c * p.L + l) * kTraceMarks + (mark)] = gtime();                         \
    } while (0)

// ---------------------------------------------------------------------------
// VPT: 16-byte column vectors per consumer thread held in registers (d <= VPT * 8 * kConsumers);
// the two-token kernels at d <= 4096 use VPT = 2, which keeps their FFN accumulators out of
// local memory
template <typename T, int NB, int HV, bool LA, bool TAB, int VPT = kMaxVPT>
__global__ void __launch_bounds__(kThreads, 1) k_decode(const __grid_constant__ Params p)
{
    extern __shared__ __align__(128) char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x, G = p.G, d = p.d, n = p.n, H = p.H, B = p.B;
    const int nvec = d >> 3;                   // 16-byte vectors per d-row
    const int hv = H >> 3;                     // 16-byte vectors per H-row
    const int fslot_bytes = 4 * d + 128;       // W1 row, W2T row, 16-byte block holding b1[j]

    // ---- carve shared memory
    Shared S;
    {
        char* q = smem;
        S.pring = q; q += (size_t)p.pred_slots * p.pred_slot_bytes;
        S.fring = q; q += (size_t)p.ffn_slots * fslot_bytes;
        S.xs = q; q += ((size_t)NB * d * sizeof(T) + 127) / 128 * 128;
        S.hs = reinterpret_cast<float*>(q); q += ((size_t)NB * H * 4 + 127) / 128 * 128;
        S.sel = reinterpret_cast<unsigned char*>(q); q += (p.max_rows + 127) / 128 * 128;   // >= 2 x 32 flags
        S.nl = reinterpret_cast<int32_t*>(q); q += ((size_t)2 * p.max_rows * 4 + 127) / 128 * 128;
        S.bias1 = reinterpret_cast<float*>(q); q += ((size_t)(H / G + 2) * 4 + 127) / 128 * 128;
        S.bias2 = reinterpret_cast<float*>(q); q += ((size_t)p.max_rows * 4 + 127) / 128 * 128;
        S.biasy = reinterpret_cast<float*>(q); q += ((size_t)(d / G + 8) * 4 + 127) / 128 * 128;
        S.red = reinterpret_cast<float*>(q); q += (2 * 4 * 8 + 2 * 8 * 2 * NB) * 4;
        S.red2 = reinterpret_cast<float*>(q); q += 8 * NB * 4;
        S.red1 = reinterpret_cast<float*>(q); q += 32 * 8 * NB * 4;
        S.misc = reinterpret_cast<float*>(q); q += 16 * 4;
        q = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(q) + 15) & ~uintptr_t(15));
        uint64_t* bars = reinterpret_cast<uint64_t*>(q);
        S.pfull = bars; S.pempty = bars + p.pred_slots;
        S.ffull = S.pempty + p.pred_slots; S.fempty = S.ffull + p.ffn_slots;
        S.flags = reinterpret_cast<volatile int*>(S.fempty + p.ffn_slots);
    }
    if (tid == 0) {
        for (int i = 0; i < p.pred_slots; ++i) { mbar_init(&S.pfull[i], 1); mbar_init(&S.pempty[i], kConsumerWarps); }
        for (int i = 0; i < p.ffn_slots; ++i) { mbar_init(&S.ffull[i], 1); mbar_init(&S.fempty[i], kConsumerWarps); }
        for (int i = 0; i < 8; ++i) S.flags[i] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // CTA c's rows of Wp1 and Wp2 (contiguous spans)
    const int a0 = split_lo(H, G, c), a1 = split_lo(H, G, c + 1);
    const int b0 = split_lo(n, G, c), b1 = split_lo(n, G, c + 1);

    // =======================================================================
    // predictor producer: streams [Wp1 rows a0..a1) then [Wp2 rows b0..b1) per layer, and
    // once a layer's copies are all issued, asks L2 to prefetch the next layer's spans so
    // HBM keeps streaming while the consumers sit in latency-bound phases.
    if (warp == kConsumerWarps) {
        if (lane == 0) {
            const uint64_t pol_first = policy_evict_first();
            int k = 0;
            for (int l = 0; l < p.L && !aborted(S, p) && !TAB; ++l) {
                for (int part = 0; part < 2; ++part) {
                    const int r0 = part ? b0 : a0, r1 = part ? b1 : a1, R = part ? p.R2 : p.R1;
                    const size_t rb = part ? (size_t)H * 2 : (size_t)d * 2;
                    const char* base = reinterpret_cast<const char*>(part ? p.layer[l].Wp2 : p.layer[l].Wp1);
                    for (int r = r0; r < r1; r += R, ++k) {
                        const int s = k % p.pred_slots;
                        if (!wait_bounded(S, p, &S.pempty[s], ((k / p.pred_slots) & 1) ^ 1, true)) goto pred_done;
                        const uint32_t bytes = (uint32_t)(min(R, r1 - r) * rb);
                        mbar_expect_tx(&S.pfull[s], bytes);
                        if (p.hot_rows > 0)
                            bulk_g2s_hint(S.pring + (size_t)s * p.pred_slot_bytes, base + (size_t)r * rb, bytes,
                                          &S.pfull[s], pol_first);
                        else
                            bulk_g2s(S.pring + (size_t)s * p.pred_slot_bytes, base + (size_t)r * rb, bytes, &S.pfull[s]);
                        S.flags[2] = k + 1;
                    }
                }
                if (l + 1 < p.L) {
                    for (int part = 0; part < 2; ++part) {
                        const int r0 = part ? b0 : a0, r1 = part ? b1 : a1;
                        const size_t rb = part ? (size_t)H * 2 : (size_t)d * 2;
                        const char* base = reinterpret_cast<const char*>(part ? p.layer[l + 1].Wp2 : p.layer[l + 1].Wp1);
                        const size_t total = (size_t)(r1 - r0) * rb;
                        for (size_t off = 0; off < total; off += 32768)
                            bulk_prefetch_l2(base + (size_t)r0 * rb + off, (uint32_t)min((size_t)32768, total - off));
                    }
                }
            }
        pred_done:
            __threadfence_block();
            S.flags[4] = 1;
        }
        return;
    }
    // =======================================================================
    // FFN producer: gathers W1[j], W2T[j] and b1[j]'s 16-byte block for every neuron the
    // consumers append to this CTA's list, as soon as it appears.
    if (warp == kConsumerWarps + 1) {
        if (lane == 0) {
            const uint64_t pol_last = policy_evict_last(), pol_first = policy_evict_first();
            // W1[j], W2T[j] and b1[j]'s 16-byte block into FFN slot s
            auto gather = [&](int s, int j, const char* w1, const char* w2, const char* bb0) {
                char* dst = S.fring + (size_t)s * fslot_bytes;
                mbar_expect_tx(&S.ffull[s], (uint32_t)(4 * d + 16));
                if (p.hot_rows > 0) {
                    // hot rows ([PI1] §5.2: the most frequently active neurons) stay in L2
                    const uint64_t pol = range_offset(j, n, G) < p.hot_rows ? pol_last : pol_first;
                    bulk_g2s_hint(dst, w1 + (size_t)j * 2 * d, (uint32_t)(2 * d), &S.ffull[s], pol);
                    bulk_g2s_hint(dst + 2 * d, w2 + (size_t)j * 2 * d, (uint32_t)(2 * d), &S.ffull[s], pol);
                } else {
                    bulk_g2s(dst, w1 + (size_t)j * 2 * d, (uint32_t)(2 * d), &S.ffull[s]);
                    bulk_g2s(dst + 2 * d, w2 + (size_t)j * 2 * d, (uint32_t)(2 * d), &S.ffull[s]);
                }
                bulk_g2s(dst + 4 * d, bb0 + (size_t)(j & ~7) * 2, 16u, &S.ffull[s]);
            };
            int k = 0;
            bool stop = false;
            for (int l = 0; l < p.L && !stop; ++l) {
                const char* w1 = reinterpret_cast<const char*>(p.layer[l].W1);
                const char* w2 = reinterpret_cast<const char*>(p.layer[l].W2T);
                const char* bb0 = reinterpret_cast<const char*>(p.layer[l].b1);
                if constexpr (TAB) {
                    // caller tables are known at launch: this CTA's slice of every layer's table,
                    // filtered exactly as the consumers filter it, streams ahead across layers as
                    // far as the FFN ring allows
                    int U = __ldcg(p.layer[l].tab_count);
                    U = U < 0 ? 0 : (U > n ? n : U);
                    const int lo = split_lo(U, G, c), hi = split_lo(U, G, c + 1);
                    for (int i = lo; i < hi && !stop; ++i) {
                        const int j = __ldcg(p.layer[l].tab + i);
                        if (j < 0 || j >= n) continue;
                        const int s = k % p.ffn_slots;
                        if (!wait_bounded(S, p, &S.fempty[s], ((k / p.ffn_slots) & 1) ^ 1, true)) { stop = true; break; }
                        gather(s, j, w1, w2, bb0);
                        S.flags[3] = ++k;
                    }
                    continue;
                }
                int issued = 0;
                unsigned long long t0 = gtime();
                while (true) {
                    const int f = S.flags[1];
                    const int avail = ((f >> 16) & 0x7fff) == (l & 0x7fff) ? (f & 0xffff) : 0;
                    if (issued < avail) {
                        __threadfence_block();
                        const int s = k % p.ffn_slots;
                        if (!wait_bounded(S, p, &S.fempty[s], ((k / p.ffn_slots) & 1) ^ 1, true)) { stop = true; break; }
                        gather(s, S.nl[(l & 1) * p.max_rows + issued], w1, w2, bb0);
                        S.flags[3] = ++k;
                        ++issued;
                        t0 = gtime();
                        continue;
                    }
                    if (S.flags[7] == l + 1) {
                        const int f2 = S.flags[1];
                        const int fin = ((f2 >> 16) & 0x7fff) == (l & 0x7fff) ? (f2 & 0xffff) : 0;
                        if (issued >= fin) break;
                        continue;
                    }
                    if (aborted(S, p)) { stop = true; break; }
                    if (gtime() - t0 > kWaitNs) { raise_abort(S, p, ERR_PIPE_TIMEOUT); stop = true; break; }
                    __nanosleep(64);
                }
            }
            __threadfence_block();
            S.flags[5] = 1;
        }
        return;
    }
    // =======================================================================
    // consumers (warps 0..7)
    uint32_t epoch = 0;
    int pk_ = 0, fk = 0;       // chunks consumed from each ring
    int rpar = 0;
    T* xs = reinterpret_cast<T*>(S.xs);
    const int R1 = p.R1, R2 = p.R2;
    bool ok = true;
    int l = 0;                 // layer whose FFN is in flight (indexes the trace rows)

    // bias slices: bp1/bp2 of predictor layer q and b2 of FFN layer f (-1: none)
    auto load_biases = [&](int q, int f) {
        if (q >= 0) {
            const T* bp1 = reinterpret_cast<const T*>(p.layer[q].bp1);
            const T* bp2 = reinterpret_cast<const T*>(p.layer[q].bp2);
            for (int i = tid; i < b1 - b0; i += kConsumers) S.bias2[i] = bp2 ? DT<T>::f(bp2[b0 + i]) : 0.f;
            if (tid < a1 - a0) S.bias1[tid] = bp1 ? DT<T>::f(bp1[a0 + tid]) : 0.f;
        }
        if (f >= 0) {
            const T* b2p = reinterpret_cast<const T*>(p.layer[f].b2);
            const int ng = d >> 2;
            const int c0 = split_lo(ng, G, c) * 4, c1 = split_lo(ng, G, c + 1) * 4;
            if (tid < c1 - c0) S.biasy[tid] = b2p ? DT<T>::f(b2p[c0 + tid]) : 0.f;
        }
    };

    // x of layer l into shared memory: the input itself for l == 0, else
    // round(u / rms(u)) from the previous layer's u = x + y.  Thread tid owns the
    // 16-byte column vectors v = tid + m*256.  For l == L the result is the output.
    auto form_x = [&](int l) {
        if (l == 0) {
            const T* xin = reinterpret_cast<const T*>(p.x_in);
#pragma unroll
            for (int m = 0; m < VPT; ++m) {
                const int v = tid + m * kConsumers;
#pragma unroll
                for (int t = 0; t < NB; ++t)
                    if (v < nvec)
                        reinterpret_cast<uint4*>(xs + (size_t)t * d)[v] =
                            __ldcg(reinterpret_cast<const uint4*>(xin + (size_t)t * d) + v);
            }
            return;
        }
        float4 uv[VPT][2][NB];
#pragma unroll
        for (int m = 0; m < VPT; ++m) {
            const int v = tid + m * kConsumers;
#pragma unroll
            for (int t = 0; t < NB; ++t) {
                if (v < nvec) {
                    const float4* up = reinterpret_cast<const float4*>(p.u + (size_t)t * d + v * 8);
                    uv[m][0][t] = __ldcg(up);
                    uv[m][1][t] = __ldcg(up + 1);
                }
            }
        }
        // rms of u from the loaded values themselves (same tree in every CTA)
        {
            float sq[NB];
#pragma unroll
            for (int t = 0; t < NB; ++t) {
                sq[t] = 0.f;
#pragma unroll
                for (int m = 0; m < VPT; ++m) {
                    const int v = tid + m * kConsumers;
                    if (v < nvec) {
                        const float4 a = uv[m][0][t], b = uv[m][1][t];
                        sq[t] = fmaf(a.x, a.x, sq[t]); sq[t] = fmaf(a.y, a.y, sq[t]);
                        sq[t] = fmaf(a.z, a.z, sq[t]); sq[t] = fmaf(a.w, a.w, sq[t]);
                        sq[t] = fmaf(b.x, b.x, sq[t]); sq[t] = fmaf(b.y, b.y, sq[t]);
                        sq[t] = fmaf(b.z, b.z, sq[t]); sq[t] = fmaf(b.w, b.w, sq[t]);
                    }
                }
                sq[t] = warp_sum(sq[t]);
                if (lane == 0) S.red2[warp * NB + t] = sq[t];
            }
            consumer_sync();
            if (tid < NB) {
                float z = 0.f;
                for (int q = 0; q < kConsumerWarps; ++q) z += S.red2[q * NB + tid];
                S.misc[tid] = 1.0f / sqrtf(z / (float)d + 1e-6f);
            }
        }
        consumer_sync();
#pragma unroll
        for (int t = 0; t < NB; ++t) {
            const float rs = S.misc[t];
#pragma unroll
            for (int m = 0; m < VPT; ++m) {
                const int v = tid + m * kConsumers;
                if (v < nvec) {
                    const float f[8] = {uv[m][0][t].x, uv[m][0][t].y, uv[m][0][t].z, uv[m][0][t].w,
                                        uv[m][1][t].x, uv[m][1][t].y, uv[m][1][t].z, uv[m][1][t].w};
                    T r8[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) r8[q] = DT<T>::r(f[q] * rs);
                    reinterpret_cast<uint4*>(xs + (size_t)t * d)[v] = *reinterpret_cast<const uint4*>(r8);
                }
            }
        }
        if (l == p.L && c == 0 && p.x_out) {
            T* xo = reinterpret_cast<T*>(p.x_out);
#pragma unroll
            for (int m = 0; m < VPT; ++m) {
                const int v = tid + m * kConsumers;
                for (int t = 0; t < B; ++t)
                    if (v < nvec)
                        reinterpret_cast<uint4*>(xo + (size_t)t * d)[v] =
                            reinterpret_cast<const uint4*>(xs + (size_t)t * d)[v];
            }
        }
    };

    // h = ReLU(Wp1 x + bp1) over this CTA's Wp1 rows [a0, a1) of the next predictor
    // layer in the ring, from the x in shared memory.  Warp w owns columns
    // [w nvec/8, (w+1) nvec/8) of every row; its lanes keep that segment of x in
    // registers as fp32 pairs, and the eight warps' partial dots of a row are added
    // in fixed order through shared memory.
    auto gemv1 = [&](int q) -> bool {
        float* hq = p.h + (size_t)(q & 1) * NB * H;
        const int seg_lo = split_lo(nvec, kConsumerWarps, warp), seg_hi = split_lo(nvec, kConsumerWarps, warp + 1);
        u64 xg[VPT][4][NB];
#pragma unroll
        for (int m = 0; m < VPT; ++m) {
            const int v = seg_lo + lane + 32 * m;
#pragma unroll
            for (int t = 0; t < NB; ++t) {
                if (v < seg_hi) {
                    const uint4 xv = reinterpret_cast<const uint4*>(xs + (size_t)t * d)[v];
                    xg[m][0][t] = Arith<T>::widen2(xv.x); xg[m][1][t] = Arith<T>::widen2(xv.y);
                    xg[m][2][t] = Arith<T>::widen2(xv.z); xg[m][3][t] = Arith<T>::widen2(xv.w);
                } else {
                    xg[m][0][t] = xg[m][1][t] = xg[m][2][t] = xg[m][3][t] = 0ull;
                }
            }
        }
        for (int r = a0; r < a1; r += R1, ++pk_) {
            const int s = pk_ % p.pred_slots;
            if (!cwait(S, p, &S.pfull[s], (pk_ / p.pred_slots) & 1)) return false;
            if (r == a0) TRACE(1);
            const uint4* slot = reinterpret_cast<const uint4*>(S.pring + (size_t)s * p.pred_slot_bytes);
            const int rows = min(R1, a1 - r);
            if constexpr (NB == 1) {
                // B = 1: four rows at a time (four independent dot chains); rows past the end
                // repeat the last row and their results are dropped.  B = 2: two rows at a time.
                constexpr int kR = 4;
                for (int rr = 0; rr < rows; rr += kR) {
                    const uint4* wp[kR];
    #pragma unroll
                    for (int u = 0; u < kR; ++u) wp[u] = slot + (size_t)min(rr + u, rows - 1) * nvec;
                    u64 cc[kR][NB];
    #pragma unroll
                    for (int u = 0; u < kR; ++u)
    #pragma unroll
                        for (int t = 0; t < NB; ++t) cc[u][t] = 0ull;
    #pragma unroll
                    for (int m = 0; m < VPT; ++m) {
                        const int v = seg_lo + lane + 32 * m;
                        if (v < seg_hi) {
    #pragma unroll
                            for (int u = 0; u < kR; ++u) {
                                const uint4 w = wp[u][v];
                                const u64 q0 = Arith<T>::widen2(w.x), q1 = Arith<T>::widen2(w.y);
                                const u64 q2 = Arith<T>::widen2(w.z), q3 = Arith<T>::widen2(w.w);
    #pragma unroll
                                for (int t = 0; t < NB; ++t) {
                                    ffma2(cc[u][t], q0, xg[m][0][t]); ffma2(cc[u][t], q1, xg[m][1][t]);
                                    ffma2(cc[u][t], q2, xg[m][2][t]); ffma2(cc[u][t], q3, xg[m][3][t]);
                                }
                            }
                        }
                    }
    #pragma unroll
                    for (int u = 0; u < kR; ++u)
    #pragma unroll
                        for (int t = 0; t < NB; ++t) {
                            const float2 e = upk(cc[u][t]);
                            const float z = warp_sum(e.x + e.y);
                            if (lane == 0 && rr + u < rows) S.red1[((rr + u) * kConsumerWarps + warp) * NB + t] = z;
                        }
                }
            } else {
                for (int rr = 0; rr < rows; rr += 2) {
                    const bool two = rr + 1 < rows;
                    const uint4* w0p = slot + (size_t)rr * nvec;
                    const uint4* w1p = slot + (size_t)(two ? rr + 1 : rr) * nvec;
                    u64 c0[NB], c1[NB];
    #pragma unroll
                    for (int t = 0; t < NB; ++t) c0[t] = c1[t] = 0ull;
    #pragma unroll
                    for (int m = 0; m < VPT; ++m) {
                        const int v = seg_lo + lane + 32 * m;
                        if (v < seg_hi) {
                            const uint4 w0 = w0p[v], w1 = w1p[v];
                            const u64 p00 = Arith<T>::widen2(w0.x), p01 = Arith<T>::widen2(w0.y);
                            const u64 p02 = Arith<T>::widen2(w0.z), p03 = Arith<T>::widen2(w0.w);
                            const u64 p10 = Arith<T>::widen2(w1.x), p11 = Arith<T>::widen2(w1.y);
                            const u64 p12 = Arith<T>::widen2(w1.z), p13 = Arith<T>::widen2(w1.w);
    #pragma unroll
                            for (int t = 0; t < NB; ++t) {
                                ffma2(c0[t], p00, xg[m][0][t]); ffma2(c0[t], p01, xg[m][1][t]);
                                ffma2(c0[t], p02, xg[m][2][t]); ffma2(c0[t], p03, xg[m][3][t]);
                                ffma2(c1[t], p10, xg[m][0][t]); ffma2(c1[t], p11, xg[m][1][t]);
                                ffma2(c1[t], p12, xg[m][2][t]); ffma2(c1[t], p13, xg[m][3][t]);
                            }
                        }
                    }
    #pragma unroll
                    for (int t = 0; t < NB; ++t) {
                        const float2 e0 = upk(c0[t]), e1 = upk(c1[t]);
                        const float z0 = warp_sum(e0.x + e0.y), z1 = warp_sum(e1.x + e1.y);
                        if (lane == 0) {
                            S.red1[(rr * kConsumerWarps + warp) * NB + t] = z0;
                            if (two) S.red1[((rr + 1) * kConsumerWarps + warp) * NB + t] = z1;
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.pempty[s]);
            consumer_sync();
            if (tid < rows * NB) {
                const int rr = tid / NB, t = tid % NB;
                float zz = 0.f;
#pragma unroll
                for (int q = 0; q < kConsumerWarps; ++q) zz += S.red1[(rr * kConsumerWarps + q) * NB + t];
                if (t < B) hq[(size_t)t * H + r + rr] = fmaxf(zz + S.bias1[r + rr - a0], 0.f);
            }
            consumer_sync();
        }
        return true;
    };

    // Logits of predictor layer q over this CTA's Wp2 rows [b0, b1), threshold, and
    // this CTA's list of selected neurons (ascending) into list buffer q & 1.  Lane
    // l keeps h's 16-byte column groups v = l + 32 i in registers as fp32 pairs.  The
    // list grows chunk by chunk and its length is published at once, so the FFN
    // producer gathers W1/W2T rows while the rest of Wp2 still streams.  Returns the
    // final length (-1 on a failed wait); the list is then published as final and its
    // length stored in the per-CTA counts of parity q & 1.
    auto gemv2 = [&](int q) -> int {
        int m = 0;
        int32_t* nl = S.nl + (q & 1) * p.max_rows;
        constexpr int kHV = HV;                // H <= 256 * HV
        // one L2 read of h per CTA (every CTA reads the same few lines: keep that traffic small)
        for (int i = tid; i < (NB * H) >> 2; i += kConsumers)
            reinterpret_cast<float4*>(S.hs)[i] = __ldcg(reinterpret_cast<const float4*>(p.h + (size_t)(q & 1) * NB * H) + i);
        consumer_sync();
        u64 hr[kHV][4][NB];
#pragma unroll
        for (int i = 0; i < kHV; ++i) {
            const int v = lane + 32 * i;
#pragma unroll
            for (int t = 0; t < NB; ++t) {
                if (v < hv) {
                    const float4* hp = reinterpret_cast<const float4*>(S.hs + (size_t)t * H + v * 8);
                    const float4 a = hp[0], b = hp[1];
                    hr[i][0][t] = pk(a.x, a.y); hr[i][1][t] = pk(a.z, a.w);
                    hr[i][2][t] = pk(b.x, b.y); hr[i][3][t] = pk(b.z, b.w);
                } else {
                    hr[i][0][t] = hr[i][1][t] = hr[i][2][t] = hr[i][3][t] = 0ull;
                }
            }
        }
        TRACE(4);
        for (int r = b0; r < b1; r += R2, ++pk_) {
            const int s = pk_ % p.pred_slots;
            // the chunk's selection flags, double-buffered by chunk: warp 0 still reads the
            // previous chunk's flags for its append while the other warps write this one's
            unsigned char* sel = S.sel + (pk_ & 1) * 32;
            if (!cwait(S, p, &S.pfull[s], (pk_ / p.pred_slots) & 1)) return -1;
            if (r == b0) TRACE(5);
            if (r == b0 + 3 * R2) TRACE(12);
            if (r + R2 >= b1) TRACE(14);
            const uint4* slot = reinterpret_cast<const uint4*>(S.pring + (size_t)s * p.pred_slot_bytes);
            const int rows = min(R2, b1 - r);
            // two rows per warp per step for independent FMA chains
            for (int rr = warp; rr < rows; rr += 2 * kConsumerWarps) {
                const int rr2 = rr + kConsumerWarps;
                const bool two = rr2 < rows;
                const uint4* w0p = slot + (size_t)rr * hv;
                const uint4* w1p = slot + (size_t)(two ? rr2 : rr) * hv;
                u64 a0[2][NB], a1[2][NB];
#pragma unroll
                for (int t = 0; t < NB; ++t) a0[0][t] = a0[1][t] = a1[0][t] = a1[1][t] = 0ull;
#pragma unroll
                for (int i = 0; i < kHV; ++i) {
                    const int v = lane + 32 * i;
                    if (v < hv) {
                        const uint4 w0 = w0p[v], w1 = w1p[v];
                        const u64 p00 = Arith<T>::widen2(w0.x), p01 = Arith<T>::widen2(w0.y);
                        const u64 p02 = Arith<T>::widen2(w0.z), p03 = Arith<T>::widen2(w0.w);
                        const u64 p10 = Arith<T>::widen2(w1.x), p11 = Arith<T>::widen2(w1.y);
                        const u64 p12 = Arith<T>::widen2(w1.z), p13 = Arith<T>::widen2(w1.w);
#pragma unroll
                        for (int t = 0; t < NB; ++t) {
                            ffma2(a0[0][t], p00, hr[i][0][t]); ffma2(a0[1][t], p01, hr[i][1][t]);
                            ffma2(a0[0][t], p02, hr[i][2][t]); ffma2(a0[1][t], p03, hr[i][3][t]);
                            ffma2(a1[0][t], p10, hr[i][0][t]); ffma2(a1[1][t], p11, hr[i][1][t]);
                            ffma2(a1[0][t], p12, hr[i][2][t]); ffma2(a1[1][t], p13, hr[i][3][t]);
                        }
                    }
                }
                bool any0 = false, any1 = false;
#pragma unroll
                for (int t = 0; t < NB; ++t) {
                    const float2 x0 = upk(a0[0][t]), x1 = upk(a0[1][t]);
                    const float2 y0 = upk(a1[0][t]), y1 = upk(a1[1][t]);
                    const float z0 = warp_sum((x0.x + x0.y) + (x1.x + x1.y));
                    const float z1 = warp_sum((y0.x + y0.y) + (y1.x + y1.y));
                    if (t < B) {
                        any0 |= (z0 + S.bias2[r + rr - b0]) > 0.f;
                        if (two) any1 |= (z1 + S.bias2[r + rr2 - b0]) > 0.f;
                    }
                }
                if (lane == 0) {
                    sel[rr] = any0;
                    if (two) sel[rr2] = any1;
                }
            }
            __syncwarp();
            if (r + R2 >= b1) TRACE(15);
            if (lane == 0) mbar_arrive(&S.pempty[s]);
            consumer_sync();
            if (r == b0 + 3 * R2) TRACE(13);
            // append this chunk's selected rows in ascending order and publish the count
            if (warp == 0) {
                for (int q0 = 0; q0 < rows; q0 += 32) {
                    const bool on = q0 + lane < rows && sel[q0 + lane];
                    const uint32_t bal = __ballot_sync(0xffffffffu, on);
                    if (on) nl[m + __popc(bal & ((1u << lane) - 1u))] = r + q0 + lane;
                    m += __popc(bal);
                }
                __syncwarp();
                if (lane == 0) {
                    __threadfence_block();
                    S.flags[1] = (q << 16) | m;
                }
            }
        }
        consumer_sync();
        {
            const int f = S.flags[1];
            m = ((f >> 16) & 0x7fff) == (q & 0x7fff) ? (f & 0xffff) : 0;   // no rows (b0 == b1): empty list
        }
        consumer_sync();
        if (tid == 0) {
            __threadfence_block();
            S.flags[7] = q + 1;                       // list q is final
            p.cta_count[(q & 1) * (G + 1) + c] = m;
        }
        TRACE(6);
        return m;
    };

    // FFN of layer l over this CTA's list (length m, buffer l & 1): FC1 (vec_dot with
    // the storage-dtype x) + bias + ReLU, then FC2 (AXPY of the neuron's W2T row) into
    // a fixed per-CTA fp32 partial, written to partial[c].
    auto ffn = [&](int l, int m) -> bool {
        const int32_t* nl = S.nl + (l & 1) * p.max_rows;
        // FC1 operand: this thread's x column vectors, packed storage pairs
        uint4 xr[VPT][NB];
#pragma unroll
        for (int a = 0; a < VPT; ++a) {
            const int v = tid + a * kConsumers;
#pragma unroll
            for (int t = 0; t < NB; ++t)
                xr[a][t] = v < nvec ? reinterpret_cast<const uint4*>(xs + (size_t)t * d)[v] : make_uint4(0, 0, 0, 0);
        }
        u64 acc[VPT][4][NB];
#pragma unroll
        for (int a = 0; a < VPT; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int t = 0; t < NB; ++t) acc[a][q][t] = 0ull;
        int i = 0;
        if constexpr (NB == 1) {
            // four neurons per step while four remain (one shared-memory reduction per quad;
            // four independent dot chains hide more latency than two)
            float* redq = S.red;
            if (p.ffn_slots >= 4) {
                for (; i + 4 <= m; i += 4, fk += 4) {
                    const char* sl[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (!cwait(S, p, &S.ffull[(fk + u) % p.ffn_slots], ((fk + u) / p.ffn_slots) & 1)) return false;
                        sl[u] = S.fring + (size_t)((fk + u) % p.ffn_slots) * fslot_bytes;
                    }
                    if (i == 0) TRACE(7);
                    float part[4][4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) part[u][0] = part[u][1] = part[u][2] = part[u][3] = 0.f;
#pragma unroll
                    for (int a = 0; a < VPT; ++a) {
                        const int v = tid + a * kConsumers;
                        if (v < nvec) {
#pragma unroll
                            for (int u = 0; u < 4; ++u) dot_mix<T>(part[u], reinterpret_cast<const uint4*>(sl[u])[v], xr[a][0]);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float v = warp_sum(sum4(part[u]));
                        if (lane == 0) redq[(rpar * 4 + u) * 8 + warp] = v;
                    }
                    consumer_sync();
                    u64 av[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float4* rp = reinterpret_cast<const float4*>(redq + (rpar * 4 + u) * 8);
                        const float4 r0 = rp[0], r1 = rp[1];
                        const float z = ((r0.x + r0.y) + (r0.z + r0.w)) + ((r1.x + r1.y) + (r1.z + r1.w));
                        const float bias = DT<T>::f(reinterpret_cast<const T*>(sl[u] + 4 * d)[nl[i + u] & 7]);
                        const float a = fmaxf(z + bias, 0.f);
                        av[u] = pk(a, a);
                    }
                    rpar ^= 1;
#pragma unroll
                    for (int a = 0; a < VPT; ++a) {
                        const int v = tid + a * kConsumers;
                        if (v < nvec) {
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const uint4 w = reinterpret_cast<const uint4*>(sl[u] + 2 * d)[v];
                                ffma2(acc[a][0][0], av[u], Arith<T>::widen2(w.x));
                                ffma2(acc[a][1][0], av[u], Arith<T>::widen2(w.y));
                                ffma2(acc[a][2][0], av[u], Arith<T>::widen2(w.z));
                                ffma2(acc[a][3][0], av[u], Arith<T>::widen2(w.w));
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0)
                        for (int u = 0; u < 4; ++u) mbar_arrive(&S.fempty[(fk + u) % p.ffn_slots]);
                }
            }
        }
        float* redp = S.red + 2 * 4 * 8;
        // the rest two at a time: one shared-memory reduction per pair
        for (; i < m; i += 2, fk += 2) {
            const bool two = i + 1 < m;
            const int s0 = fk % p.ffn_slots, s1 = (fk + 1) % p.ffn_slots;
            if (!cwait(S, p, &S.ffull[s0], (fk / p.ffn_slots) & 1)) return false;
            if (two && !cwait(S, p, &S.ffull[s1], ((fk + 1) / p.ffn_slots) & 1)) return false;
            if (i == 0) TRACE(7);
            const char* sl0 = S.fring + (size_t)s0 * fslot_bytes;
            const char* sl1 = S.fring + (size_t)(two ? s1 : s0) * fslot_bytes;
            float part[2][NB][4];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int t = 0; t < NB; ++t) part[u][t][0] = part[u][t][1] = part[u][t][2] = part[u][t][3] = 0.f;
#pragma unroll
            for (int a = 0; a < VPT; ++a) {
                const int v = tid + a * kConsumers;
                if (v < nvec) {
                    const uint4 w0 = reinterpret_cast<const uint4*>(sl0)[v];
                    const uint4 w1 = reinterpret_cast<const uint4*>(sl1)[v];
#pragma unroll
                    for (int t = 0; t < NB; ++t) {
                        dot_mix<T>(part[0][t], w0, xr[a][t]);
                        dot_mix<T>(part[1][t], w1, xr[a][t]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int t = 0; t < NB; ++t) {
                    const float v = warp_sum(sum4(part[u][t]));
                    if (lane == 0) redp[((rpar * 8 + warp) * 2 + u) * NB + t] = v;
                }
            consumer_sync();
            u64 av[2][NB];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const char* sl = u ? sl1 : sl0;
                const int j = nl[u ? (two ? i + 1 : i) : i];
                const float bias = DT<T>::f(reinterpret_cast<const T*>(sl + 4 * d)[j & 7]);
#pragma unroll
                for (int t = 0; t < NB; ++t) {
                    float z = 0.f;
#pragma unroll
                    for (int q = 0; q < kConsumerWarps; ++q) z += redp[((rpar * 8 + q) * 2 + u) * NB + t];
                    float a = fmaxf(z + bias, 0.f);
                    if (u == 1 && !two) a = 0.f;
                    av[u][t] = pk(a, a);
                }
            }
            rpar ^= 1;
#pragma unroll
            for (int a = 0; a < VPT; ++a) {
                const int v = tid + a * kConsumers;
                if (v < nvec) {
                    const uint4 w0 = reinterpret_cast<const uint4*>(sl0 + 2 * d)[v];
                    const uint4 w1 = reinterpret_cast<const uint4*>(sl1 + 2 * d)[v];
                    const u64 q00 = Arith<T>::widen2(w0.x), q01 = Arith<T>::widen2(w0.y);
                    const u64 q02 = Arith<T>::widen2(w0.z), q03 = Arith<T>::widen2(w0.w);
#pragma unroll
                    for (int t = 0; t < NB; ++t) {
                        ffma2(acc[a][0][t], av[0][t], q00); ffma2(acc[a][1][t], av[0][t], q01);
                        ffma2(acc[a][2][t], av[0][t], q02); ffma2(acc[a][3][t], av[0][t], q03);
                    }
                    if (two) {
                        const u64 q10 = Arith<T>::widen2(w1.x), q11 = Arith<T>::widen2(w1.y);
                        const u64 q12 = Arith<T>::widen2(w1.z), q13 = Arith<T>::widen2(w1.w);
#pragma unroll
                        for (int t = 0; t < NB; ++t) {
                            ffma2(acc[a][0][t], av[1][t], q10); ffma2(acc[a][1][t], av[1][t], q11);
                            ffma2(acc[a][2][t], av[1][t], q12); ffma2(acc[a][3][t], av[1][t], q13);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&S.fempty[s0]);
                if (two) mbar_arrive(&S.fempty[s1]);
            }
            if (!two) fk -= 1;               // only one slot consumed
        }
#pragma unroll
        for (int a = 0; a < VPT; ++a) {
            const int v = tid + a * kConsumers;
            if (v < nvec) {
#pragma unroll
                for (int t = 0; t < NB; ++t) {
                    float4* dst = reinterpret_cast<float4*>(p.partial + ((size_t)c * NB + t) * d + v * 8);
                    const float2 e0 = upk(acc[a][0][t]), e1 = upk(acc[a][1][t]);
                    const float2 e2 = upk(acc[a][2][t]), e3 = upk(acc[a][3][t]);
                    __stcg(dst, make_float4(e0.x, e0.y, e1.x, e1.y));
                    __stcg(dst + 1, make_float4(e2.x, e2.y, e3.x, e3.y));
                }
            }
        }
        TRACE(8);
        return true;
    };

    // y of layer l for this CTA's column groups: b2 + the G partials added in fixed
    // order, and u = x + y for the next layer (y itself kept for the last layer).
    auto reduce = [&](int l) {
        const int NG = d >> 2;                         // float4 column groups
        const int g0 = split_lo(NG, G, c), g1 = split_lo(NG, G, c + 1);
        const int tasks = (g1 - g0) * NB;
        for (int task = warp; task < tasks; task += kConsumerWarps) {
            const int g = g0 + task / NB, t = task % NB;
            float4 v[kMaxG / 32];
#pragma unroll
            for (int i = 0; i < kMaxG / 32; ++i) {
                const int s = lane + 32 * i;
                v[i] = s < G ? __ldcg(reinterpret_cast<const float4*>(p.partial + ((size_t)s * NB + t) * d + g * 4))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float4 a = v[0];
#pragma unroll
            for (int i = 1; i < kMaxG / 32; ++i) { a.x += v[i].x; a.y += v[i].y; a.z += v[i].z; a.w += v[i].w; }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                a.x += __shfl_xor_sync(0xffffffffu, a.x, o);
                a.y += __shfl_xor_sync(0xffffffffu, a.y, o);
                a.z += __shfl_xor_sync(0xffffffffu, a.z, o);
                a.w += __shfl_xor_sync(0xffffffffu, a.w, o);
            }
            if (lane == 0 && t < B) {
                float yv[4] = {a.x, a.y, a.z, a.w};
                float uv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int col = g * 4 + q;
                    yv[q] += S.biasy[col - g0 * 4];
                    uv[q] = DT<T>::f(xs[(size_t)t * d + col]) + yv[q];
                }
                if (l == p.L - 1)
                    *reinterpret_cast<float4*>(p.y + (size_t)t * d + g * 4) = make_float4(yv[0], yv[1], yv[2], yv[3]);
                __stcg(reinterpret_cast<float4*>(p.u + (size_t)t * d + g * 4), make_float4(uv[0], uv[1], uv[2], uv[3]));
            }
        }
    };

    // neuron table of layer l: this CTA's ascending entries (list buffer l & 1) at
    // their global positions, from every CTA's count of that list; CTA 0 stores the
    // total.  The last consumer warp only (it has no reduction task at B = 1 when a
    // CTA owns fewer than 8 column groups, so the count loads overlap the reduction).
    auto table = [&](int l, int m) {
        if (warp != kConsumerWarps - 1) return;
        const int32_t* cnt = p.cta_count + (l & 1) * (G + 1);
        const int32_t* nl = S.nl + (l & 1) * p.max_rows;
        int off = 0, tot = 0;
        for (int g = lane; g < G; g += 32) {
            const int v = __ldcg(cnt + g);
            off += g < c ? v : 0;
            tot += v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            off += __shfl_xor_sync(0xffffffffu, off, o);
            tot += __shfl_xor_sync(0xffffffffu, tot, o);
        }
        int32_t* idx = p.layer[l].idx;
        for (int i = lane; i < m; i += 32) idx[off + i] = nl[i];
        if (c == 0 && lane == 0 && p.counts) p.counts[l] = tot;
    };

    // caller-tables mode: this CTA's equal slice of layer l's table into list buffer l & 1
    // (entries outside [0, n) are skipped and latched, the length is clamped to [0, n) and
    // latched), published as final for the FFN producer; returns the list length
    auto take_table = [&](int l) -> int {
        int32_t* nl = S.nl + (l & 1) * p.max_rows;
        int m = 0;
        if (warp == 0) {
            int U = __ldcg(p.layer[l].tab_count);
            if (U < 0 || U > n) {
                if (c == 0 && lane == 0) atomicOr(p.err, ERR_COUNT_CLAMPED);
                U = U < 0 ? 0 : n;
            }
            const int lo = split_lo(U, G, c), hi = split_lo(U, G, c + 1);
            for (int i0 = lo; i0 < hi; i0 += 32) {
                const int i = i0 + lane;
                const int j = i < hi ? __ldcg(p.layer[l].tab + i) : -1;
                const bool bad = i < hi && (j < 0 || j >= n);
                if (bad) atomicOr(p.err, ERR_IDX_RANGE);
                const bool on = i < hi && !bad;
                const uint32_t bal = __ballot_sync(0xffffffffu, on);
                if (on) nl[m + __popc(bal & ((1u << lane) - 1u))] = j;
                m += __popc(bal);
            }
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                S.flags[1] = (l << 16) | m;
                S.flags[7] = l + 1;                    // the list of layer l is final
                if (c == 0 && p.counts) p.counts[l] = U;
                S.misc[15] = __int_as_float(m);
            }
        }
        consumer_sync();
        return __float_as_int(S.misc[15]);
    };

    if constexpr (TAB) {
        // Per layer l: x_l, this CTA's slice of the caller's table, FFN -> partial | grid barrier
        //              y_l, u_l                                                      | grid barrier
        for (l = 0; l < p.L && ok; ++l) {
            load_biases(-1, l);
            form_x(l);
            consumer_sync();
            TRACE(0);
            const int m = take_table(l);
            TRACE(6);
            if (!ffn(l, m)) { ok = false; break; }
            if (!grid_barrier(S, p, epoch)) { ok = false; break; }
            TRACE(9);
            reduce(l);
            TRACE(10);
            if (!grid_barrier(S, p, epoch)) { ok = false; break; }
            TRACE(11);
        }
    } else if constexpr (!LA) {
        // Per layer l: A  x_l, h_l (Wp1 rows)            | grid barrier
        //              B  logits_l, list_l, FFN_l -> partial | grid barrier
        //              D  y_l, u_l, table_l                | grid barrier
        for (l = 0; l < p.L && ok; ++l) {
            load_biases(l, l);
            form_x(l);
            consumer_sync();
            TRACE(0);
            if (!gemv1(l)) { ok = false; break; }
            TRACE(2);
            if (!grid_barrier(S, p, epoch)) { ok = false; break; }
            TRACE(3);
            const int m = gemv2(l);
            if (m < 0) { ok = false; break; }
            if (!ffn(l, m)) { ok = false; break; }
            if (!grid_barrier(S, p, epoch)) { ok = false; break; }
            TRACE(9);
            table(l, m);
            reduce(l);
            TRACE(10);
            if (!grid_barrier(S, p, epoch)) { ok = false; break; }
            TRACE(11);
        }
    } else {
        // Look-ahead: the neuron set of layer l+1 is predicted from x_l, so each layer
        // has two grid barriers and the FFN rows of layer l are gathered while layer
        // l-1's grid still runs.  Prologue: x_0, h_0 | barrier | logits_0, list_0.
        // Per layer l: x_l, h_{l+1}, FFN_l -> partial      | grid barrier
        //              logits_{l+1}, list_{l+1}; y_l, u_l, table_l | grid barrier
        int m = 0;
        load_biases(0, -1);
        form_x(0);
        consumer_sync();
        if (!gemv1(0) || !grid_barrier(S, p, epoch)) ok = false;
        if (ok) {
            m = gemv2(0);
            if (m < 0) ok = false;
        }
        for (l = 0; l < p.L && ok; ++l) {
            const bool next = l + 1 < p.L;
            load_biases(next ? l + 1 : -1, l);
            if (l > 0) form_x(l);
            consumer_sync();
            TRACE(0);
            if (next && !gemv1(l + 1)) { ok = false; break; }
            TRACE(2);
            if (!ffn(l, m)) { ok = false; break; }
            if (!grid_barrier(S, p, epoch)) { ok = false; break; }
            TRACE(3);
            const int m_next = next ? gemv2(l + 1) : 0;
            if (m_next < 0) { ok = false; break; }
            table(l, m);
            reduce(l);
            m = m_next;
            TRACE(10);
            if (!grid_barrier(S, p, epoch)) { ok = false; break; }
            TRACE(11);
        }
    }
    if (ok) form_x(p.L);

    // ---- drain: never leave a bulk copy in flight
    if (!ok) {
        if (tid == 0) {
            const unsigned long long t0 = gtime();
            while (!(S.flags[4] && S.flags[5]) && gtime() - t0 < kWaitNs) {}
            const int pi = S.flags[2], fi = S.flags[3];
            for (int k = pk_; k < pi; ++k) {
                const unsigned long long t1 = gtime();
                while (!mbar_try(&S.pfull[k % p.pred_slots], (k / p.pred_slots) & 1) && gtime() - t1 < kWaitNs) {}
            }
            for (int k = fk; k < fi; ++k) {
                const unsigned long long t1 = gtime();
                while (!mbar_try(&S.ffull[k % p.ffn_slots], (k / p.ffn_slots) & 1) && gtime() - t1 < kWaitNs) {}
            }
        }
    }
}

// ---------------------------------------------------------------------------
unsigned long long* g_trace = nullptr;
size_t g_trace_bytes = 0;
unsigned long long g_wait_ns = kWaitNs;     // spffn_set_wait_test
uint32_t g_bar_extra = 0;
int g_hot_rows = 0;                        // spffn_set_l2_hot_rows

int pow2_floor(int v) {
    int r = 1;
    while (r * 2 <= v) r *= 2;
    return r;
}

struct Geometry {
    int pred_slots, pred_slot_bytes, ffn_slots, R1, R2, max_rows;
    size_t smem;
};

template <typename T, int NB>
Geometry geometry(const spffn_config& c, int G, bool lookahead, bool tables = false) {
    Geometry g;
    const int budget = 227 * 1024;
    g.pred_slot_bytes = 32 * 1024;
    g.R1 = max(1, pow2_floor(g.pred_slot_bytes / (2 * c.d)));
    g.R2 = max(1, pow2_floor(g.pred_slot_bytes / (2 * c.H)));
    if (g.R2 > 32) g.R2 = 32;
    if (g.R1 > 32) g.R1 = 32;
    g.max_rows = (c.n + G - 1) / G + 1;
    size_t fixed = 0;
    fixed += ((size_t)NB * c.d * sizeof(T) + 127) / 128 * 128;      // xs
    fixed += ((size_t)NB * c.H * 4 + 127) / 128 * 128;              // hs
    fixed += (g.max_rows + 127) / 128 * 128;                         // sel
    fixed += ((size_t)2 * g.max_rows * 4 + 127) / 128 * 128;         // nl, two lists
    fixed += ((size_t)(c.H / G + 2) * 4 + 127) / 128 * 128;          // bias1
    fixed += ((size_t)g.max_rows * 4 + 127) / 128 * 128;             // bias2
    fixed += ((size_t)(c.d / G + 8) * 4 + 127) / 128 * 128;          // biasy
    fixed += (2 * 4 * 8 + 2 * 8 * 2 * NB) * 4 + 8 * NB * 4 + 32 * 8 * NB * 4 + 16 * 4 + 16;
    fixed += 8 * (2 * 8 + 2 * 8) + 8 * 8 + 128;                      // barriers + flags + slack
    const size_t fslot = 4 * (size_t)c.d + 128;
    // three predictor slots feed the logits GEMV as fast as four (its chunk rate is set
    // inside the SM), so the rest of shared memory goes to FFN slots: more of a CTA's
    // rows are resident when its list is final.  Caller tables stream no predictor.
    g.pred_slots = tables ? 1 : 3;
    g.ffn_slots = (tables || lookahead) ? 10 : 8;
    auto total = [&]() { return fixed + (size_t)g.pred_slots * g.pred_slot_bytes + g.ffn_slots * fslot; };
    while (total() > (size_t)budget && g.ffn_slots > 3) --g.ffn_slots;
    while (total() > (size_t)budget && g.pred_slots > 3) --g.pred_slots;
    while (total() > (size_t)budget && g.ffn_slots > 2) --g.ffn_slots;
    while (total() > (size_t)budget && g.pred_slots > 2) --g.pred_slots;
    g.smem = total();
    return g;
}

template <typename T, int NB, int HV, bool LA, bool TAB = false, int VPT = kMaxVPT>
cudaError_t launch_t(spffn_ctx* const* layers, int L, const void* x_in, int B, void* x_out, float* y,
                     int32_t* counts, cudaStream_t st, const int32_t* const* tabs = nullptr,
                     const int32_t* const* tab_counts = nullptr)
{
    const spffn_ctx& c0 = *layers[0];
    const int G = c0.lay.S;
    const bool tables = TAB;
    if (TAB != (tabs != nullptr)) return cudaErrorInvalidValue;
    Geometry g = geometry<T, NB>(c0.cfg, G, LA, tables);
    if (g.smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    Params p;          // host staging copy (per call: concurrent callers on other stacks stay independent);
                       // the launch copies it into the kernel's parameter space
    memset(&p, 0, sizeof(p));
    p.L = L; p.B = B; p.d = c0.cfg.d; p.n = c0.cfg.n; p.H = c0.cfg.H; p.G = G;
    p.x_in = x_in; p.x_out = x_out; p.y = y; p.counts = counts;
    Ctl* ctl = c0.ctl();
    p.bar = &ctl->barrier[0];
    p.err = &ctl->err;
    p.abort = &ctl->barrier[1];
    p.cta_count = c0.ctacnt();
    p.h = c0.h();
    p.partial = c0.partial();
    p.u = c0.ybuf();
    p.pred_slots = g.pred_slots; p.pred_slot_bytes = g.pred_slot_bytes; p.ffn_slots = g.ffn_slots;
    p.R1 = g.R1; p.R2 = g.R2; p.max_rows = g.max_rows;
    p.trace = (g_trace && g_trace_bytes >= (size_t)G * L * kTraceMarks * 8) ? g_trace : nullptr;
    p.wait_ns = g_wait_ns;
    p.bar_extra = g_bar_extra;
    p.hot_rows = g_hot_rows;
    for (int l = 0; l < L; ++l) {
        const spffn_ctx& c = *layers[l];
        p.layer[l] = LayerW{c.w.W1, c.w.b1, c.w.W2T, c.w.b2, c.w.Wp1, c.w.bp1, c.w.Wp2, c.w.bp2, c.idx(),
                            tables ? tabs[l] : nullptr, tables ? tab_counts[l] : nullptr};
    }
    cudaError_t e = cudaFuncSetAttribute(k_decode<T, NB, HV, LA, TAB, VPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.smem);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(&ctl->barrier[0], 0, 2 * sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = g.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_decode<T, NB, HV, LA, TAB, VPT>, p);
}

// the two-token kernels at d <= 4096 keep two column vectors per thread (VPT = 2)
template <typename T, int NB, int HV>
cudaError_t launch_vpt(bool lookahead, bool narrow, spffn_ctx* const* layers, int L, const void* x_in, int B,
                       void* x_out, float* y, int32_t* counts, cudaStream_t st)
{
    if constexpr (NB == 2) {
        if (narrow)
            return lookahead ? launch_t<T, NB, HV, true, false, 2>(layers, L, x_in, B, x_out, y, counts, st)
                             : launch_t<T, NB, HV, false, false, 2>(layers, L, x_in, B, x_out, y, counts, st);
    }
    return lookahead ? launch_t<T, NB, HV, true>(layers, L, x_in, B, x_out, y, counts, st)
                     : launch_t<T, NB, HV, false>(layers, L, x_in, B, x_out, y, counts, st);
}

}  // namespace

bool fused_tables_supported(spffn_ctx* const* layers, int L, int B)
{
    if (L < 1 || L > kMaxFusedLayers || B < 1 || B > 2) return false;
    const spffn_config& c0 = layers[0]->cfg;
    if (c0.d > kMaxVPT * 8 * kConsumers) return false;
    if (layers[0]->lay.S > kMaxG || layers[0]->lay.S != layers[0]->num_sms) return false;
    for (int l = 1; l < L; ++l) {
        const spffn_config& c = layers[l]->cfg;
        if (c.d != c0.d || c.n != c0.n || c.dtype != c0.dtype) return false;
    }
    const Geometry g = c0.dtype == SPFFN_BF16 ? geometry<__nv_bfloat16, 2>(c0, layers[0]->lay.S, false, true)
                                          : geometry<__half, 2>(c0, layers[0]->lay.S, false, true);
    return g.smem <= 227 * 1024;
}

bool fused_decode_supported(spffn_ctx* const* layers, int L, int B)
{
    if (L < 1 || L > kMaxFusedLayers || B < 1 || B > 2) return false;
    const spffn_config& c0 = layers[0]->cfg;
    if (c0.d > kMaxVPT * 8 * kConsumers) return false;
    if (layers[0]->lay.S > kMaxG) return false;
    if (c0.n / 32 > kMaxMaskWords) return false;
    if (c0.H > 2048 || (B == 2 && c0.H > 1024)) return false;   // h lives in registers
    for (int l = 1; l < L; ++l) {
        const spffn_config& c = layers[l]->cfg;
        if (c.d != c0.d || c.n != c0.n || c.H != c0.H || c.dtype != c0.dtype) return false;
    }
    if (layers[0]->lay.S != layers[0]->num_sms) return false;
    return true;
}

void set_trace(void* buf, size_t bytes)
{
    g_trace = static_cast<unsigned long long*>(buf);
    g_trace_bytes = buf ? bytes : 0;
}

int trace_marks() { return kTraceMarks; }

void set_wait_test(unsigned long long limit_ns, bool unmeetable_barrier)
{
    g_wait_ns = limit_ns ? limit_ns : kWaitNs;
    g_bar_extra = unmeetable_barrier ? 1u : 0u;
}

void set_l2_hot_rows(int rows) { g_hot_rows = rows > 0 ? rows : 0; }
int l2_hot_rows() { return g_hot_rows; }

unsigned long long wait_test_ns() { return g_wait_ns; }
uint32_t wait_test_bar_extra() { return g_bar_extra; }
void* trace_buffer(size_t need) { return (g_trace && g_trace_bytes >= need) ? g_trace : nullptr; }
size_t trace_bytes() { return g_trace ? g_trace_bytes : 0; }

cudaError_t launch_fused_decode(spffn_ctx* const* layers, int L, const void* x_in, int B, void* x_out, float* y,
                                int32_t* counts, bool lookahead, cudaStream_t st)
{
    const bool bf = layers[0]->cfg.dtype == SPFFN_BF16;
    const int hvn = (layers[0]->cfg.H + 255) / 256;
    const bool narrow = layers[0]->cfg.d <= 2 * 8 * kConsumers;      // two column vectors per thread
#define SPFFN_GO(TT, NBV, HVV) \
    return launch_vpt<TT, NBV, HVV>(lookahead, narrow, layers, L, x_in, B, x_out, y, counts, st)
#define SPFFN_HV(TT, NBV)                                     \
    if (hvn <= 1) SPFFN_GO(TT, NBV, 1);                       \
    if (hvn <= 2) SPFFN_GO(TT, NBV, 2);                       \
    if (hvn <= 4) SPFFN_GO(TT, NBV, 4);                       \
    if (NBV == 1) SPFFN_GO(TT, 1, 8);                         \
    return cudaErrorInvalidValue;
    if (B == 1) {
        if (bf) { SPFFN_HV(__nv_bfloat16, 1) } else { SPFFN_HV(__half, 1) }
    }
    if (bf) { SPFFN_HV(__nv_bfloat16, 2) } else { SPFFN_HV(__half, 2) }
#undef SPFFN_HV
#undef SPFFN_GO
}

cudaError_t launch_fused_tables(spffn_ctx* const* layers, int L, const void* x_in, int B,
                                const int32_t* const* tabs, const int32_t* const* tab_counts, void* x_out,
                                float* y, int32_t* counts, cudaStream_t st)
{
    // the logits GEMV does not run: any hidden width fits (HV only sizes its registers)
    const bool bf = layers[0]->cfg.dtype == SPFFN_BF16;
    if (B == 1) {
        return bf ? launch_t<__nv_bfloat16, 1, 1, false, true>(layers, L, x_in, B, x_out, y, counts, st, tabs, tab_counts)
                  : launch_t<__half, 1, 1, false, true>(layers, L, x_in, B, x_out, y, counts, st, tabs, tab_counts);
    }
    if (layers[0]->cfg.d <= 2 * 8 * kConsumers)
        return bf ? launch_t<__nv_bfloat16, 2, 1, false, true, 2>(layers, L, x_in, B, x_out, y, counts, st, tabs, tab_counts)
                  : launch_t<__half, 2, 1, false, true, 2>(layers, L, x_in, B, x_out, y, counts, st, tabs, tab_counts);
    return bf ? launch_t<__nv_bfloat16, 2, 1, false, true>(layers, L, x_in, B, x_out, y, counts, st, tabs, tab_counts)
              : launch_t<__half, 2, 1, false, true>(layers, L, x_in, B, x_out, y, counts, st, tabs, tab_counts);
}

}  // namespace spffn
