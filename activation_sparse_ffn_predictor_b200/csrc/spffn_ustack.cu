// Persistent whole-stack decode on the union tensor-core path (3 <= B <= 128).
//
// With B tokens the union of the per-token neuron sets makes every step of a
// layer a dense contraction over gathered rows ([SPX] on batch size: the sets
// are OR-ed over the batch).  One cooperative launch runs the whole stack; per
// layer l (x_l: the layer input, storage dtype, in HBM):
//
//   P0  h = ReLU(Wp1 x_l + bp1)          D[H x N1]   split-K, -> hsplit (hi/lo) | grid barrier 0
//   P1  l = Wp2 h + bp2, l > 0 -> mask   D[n x N2]                             | grid barrier 1
//   C   neuron table (ascending) from the mask words: every CTA expands all of
//       it into its own copy (L2-resident) and writes its slice of the table
//       the caller reads; no barrier: a CTA's gathers read only its own copy
//   P2  a = ReLU(W1[table] x_l + b1)     D[U x N1]   split-K, -> asplit (hi/lo) | grid barrier 2
//   P3  y = W2T[table]^T a + b2          D[d x N2]   split-K, u = x_l + y and
//       the per-tile sums of squares of u                                     | grid barrier 3
//   X   x_{l+1} = round(u / sqrt(mean(u^2) + 1e-6)), every CTA its slice      | grid barrier 4
//
// N1 = round16(B) columns (tokens); N2 = 2 N1: fp32 activations (h, a) enter the
// 16-bit MMA as a hi/lo pair of the storage dtype, whose two column halves the
// epilogue adds.
//
// One CTA per SM, warp-specialised, one continuous shared-memory ring:
// - warp 0 (one lane) issues TMA 2-D tile loads (no multicast): the weight tiles
//   of P0/P1 (Wp1, Wp2) and the activation tiles of every phase.  The weights do
//   not depend on the data, so they are issued as soon as a stage is free; an
//   activation tile whose producer phase is still running elsewhere is deferred
//   (up to one ring of stages) until its grid barrier completes, so HBM keeps
//   streaming weights across the barrier;
// - warps 6..9 gather the table rows of W1 (P2, K-major) and W2T (P3, MN-major)
//   with 16-byte cp.async into the 128-byte swizzled image the MMA reads; the
//   rows of P3 depend only on the table, so they too run ahead across barrier 3;
// - warp 1 (one lane) issues tcgen05.mma into a double-buffered TMEM accumulator;
// - warps 2..5 read TMEM, write split-K partials, and the last CTA on a tile
//   (atomic ticket) reduces the splits in fixed order; they also run C and X and
//   arrive on the grid barriers.
// Every wait is bounded (globaltimer); on expiry the CTA latches an error, raises
// the grid-wide abort flag, stops issuing copies, drains what it issued and
// returns.  Results are deterministic (fixed split and reduction orders).
#include <cuda.h>
#include <algorithm>
#include <cstring>
#include <new>
#include "spffn_internal.cuh"
#include "spffn_umma.cuh"
#include "spffn_fused.cuh"
#include "spffn_union.cuh"

namespace spffn {
namespace {
using namespace um;

constexpr int kSThreads = 320;
constexpr int kSMaxLayers = 64;       // per launch (kernel parameter space)
constexpr int kSBM = 128;
constexpr int kSBK = 64;
constexpr int kSMaxStages = 8;
constexpr int kSLag = 4;              // gather groups per thread: up to kSLag - 1 in flight (stages >= kSLag)
constexpr int kSBarriers = 5;         // grid barriers per layer
constexpr int kSTraceMarks = 16;
constexpr unsigned long long kSDrainNs = 20000000ull;

struct SLayer {
    const void *W1, *b1, *W2T, *b2, *bp1, *bp2;
    int32_t* idx;
};

struct alignas(64) SParams {
    CUtensorMap tmWp1[kSMaxLayers];   // [H][d], box {64, 128}
    CUtensorMap tmWp2[kSMaxLayers];   // [n][H], box {64, 128}
    CUtensorMap tmX[3];               // x_in, xbuf[0], xbuf[1]: [B][d], box {64, N1}
    CUtensorMap tmH;                  // hsplit [N2][H], box {64, N2}
    CUtensorMap tmA;                  // asplit [N2][n], box {64, N2}
    SLayer layer[kSMaxLayers];
    int L, B, d, n, H, G, dtype, N1, N2;
    int stages, stage_bytes, tmem_cols;
    const void* x_in;
    void* xbuf[2];
    void* x_out;
    float* y;
    int32_t* counts;
    void* hsplit;          // [N2][H]: rows 0..N1-1 hi, N1..N2-1 lo
    void* asplit;          // [N2][n]
    uint32_t* mask;        // [n / 32]
    float* partial;        // [units][128][N]
    uint32_t* tickets;     // [tiles]
    float* u;              // [B][d]
    float* ss;             // [d / 128][B]
    int32_t* ptab;         // [G][n]: each CTA's own copy of the layer's neuron table
    uint32_t* bar;
    uint32_t* abort;
    uint32_t* err;
    unsigned long long wait_ns;  // limit of a grid-barrier wait (other waits: kUWaitNs)
    uint32_t bar_extra;          // arrivals a grid barrier expects beyond G (0; 1 only under the wait test)
    unsigned long long* trace;   // optional [G][L][kSTraceMarks]
};
static_assert(sizeof(SParams) <= 32000, "kernel parameter space");

// the work of one phase: units u = (tile, split) with K blocks [kb0, kb1)
struct SPlan {
    int mode, N, M, K, tiles, kblocks, splits, units;
};

__device__ __forceinline__ SPlan splan(const SParams& p, int mode, int U) {
    SPlan q;
    q.mode = mode;
    if (mode == 0) { q.M = p.H; q.K = p.d; q.N = p.N1; }
    else if (mode == 1) { q.M = p.n; q.K = p.H; q.N = p.N2; }
    else if (mode == 2) { q.M = U; q.K = p.d; q.N = p.N1; }
    else { q.M = p.d; q.K = U; q.N = p.N2; }
    q.tiles = (q.M + kSBM - 1) / kSBM;
    q.kblocks = (q.K + kSBK - 1) / kSBK;
    if (mode == 1) {
        q.splits = 1;
    } else {
        const int s = q.tiles > 0 ? p.G / q.tiles : 1;
        q.splits = max(1, min(s, q.kblocks));
    }
    q.units = q.tiles * q.splits;
    return q;
}
__device__ __forceinline__ int kb_lo(const SPlan& q, int sp) { return (int)((long long)sp * q.kblocks / q.splits); }

__device__ __forceinline__ uint32_t gb_target(const SParams& p, int l, int b) {
    return (uint32_t)(l * kSBarriers + b + 1) * ((uint32_t)p.G + p.bar_extra);
}
__device__ __forceinline__ uint32_t ld_acq(const uint32_t* a) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
// wait until at most n of this thread's cp.async groups are pending (n = 2..6)
__device__ __forceinline__ void cp_async_wait_n(int n) {
    switch (n) {
        case 2: cp_async_wait<2>(); break;
        case 3: cp_async_wait<3>(); break;
        case 4: cp_async_wait<4>(); break;
        case 5: cp_async_wait<5>(); break;
        default: cp_async_wait<6>(); break;
    }
}
__device__ __forceinline__ void gather_sync() { asm volatile("bar.sync 3, 128;" ::: "memory"); }

struct SShared {
    uint64_t full[kSMaxStages], empty[kSMaxStages], tfull[2], tempty[2], done;
    int abort;           // this CTA gives up
    int flagU;           // layer + 1 once U of that layer is published
    int U[2];            // by layer parity
    int gok[2], eok[2], last;
    uint32_t tmem;
    int scan[128];
    float red[4][16];
    float rs[128];
    float sst[128];
};

__device__ __forceinline__ bool aborted(const SParams& p, const SShared* S) {
    return *(volatile int*)&S->abort != 0 || *(volatile uint32_t*)p.abort != 0;
}
__device__ __forceinline__ void raise_abort(const SParams& p, SShared* S, uint32_t bits) {
    *(volatile int*)&S->abort = 1;
    atomicOr(p.err, bits);
    atomicExch(p.abort, 1u);
}
// bounded wait for a grid barrier; false on timeout or abort
__device__ __forceinline__ bool gb_wait(const SParams& p, SShared* S, uint32_t target) {
    if (ld_acq(p.bar) >= target) return true;
    const unsigned long long t0 = now_ns();
    while (ld_acq(p.bar) < target) {
        if (aborted(p, S)) { *(volatile int*)&S->abort = 1; return false; }
        if (now_ns() - t0 > p.wait_ns) { raise_abort(p, S, ERR_BARRIER_TIMEOUT); return false; }
    }
    return true;
}
__device__ __forceinline__ bool mb_wait(const SParams& p, SShared* S, uint64_t* b, uint32_t parity) {
    if (ub_try(b, parity)) return true;
    const unsigned long long t0 = now_ns();
    while (!ub_try(b, parity)) {
        if (aborted(p, S)) { *(volatile int*)&S->abort = 1; return false; }
        if (now_ns() - t0 > kUWaitNs) { raise_abort(p, S, ERR_PIPE_TIMEOUT); return false; }
    }
    return true;
}
// U of layer l, published by this CTA's epilogue after the compaction
__device__ __forceinline__ int wait_U(const SParams& p, SShared* S, int l) {
    if (*(volatile int*)&S->flagU >= l + 1) return *(volatile int*)&S->U[l & 1];
    const unsigned long long t0 = now_ns();
    while (*(volatile int*)&S->flagU < l + 1) {
        if (aborted(p, S)) { *(volatile int*)&S->abort = 1; return -1; }
        if (now_ns() - t0 > kUWaitNs) { raise_abort(p, S, ERR_PIPE_TIMEOUT); return -1; }
    }
    return *(volatile int*)&S->U[l & 1];
}

template <typename T>
__device__ __forceinline__ float ldf(const void* base, int i) {
    return base ? DT<T>::f(reinterpret_cast<const T*>(base)[i]) : 0.f;
}

// the layer input x_l and the buffer the chaining of layer l writes
__device__ __forceinline__ int x_map(int l) { return l == 0 ? 0 : 1 + ((l - 1) & 1); }
__device__ __forceinline__ const void* x_ptr(const SParams& p, int l) { return l == 0 ? p.x_in : p.xbuf[(l - 1) & 1]; }

#define STRACE(mark)                                                                                 \
    do {                                                                                             \
        if (p.trace) p.trace[((size_t)blockIdx.x * p.L + l) * kSTraceMarks + (mark)] = now_ns();     \
    } while (0)

template <typename T>
__global__ void __launch_bounds__(kSThreads, 1) k_ustack(const __grid_constant__ SParams p)
{
    extern __shared__ __align__(1024) char usm[];
    char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(usm) + 1023) & ~uintptr_t(1023));
    const int SB = p.stage_bytes, NS = p.stages;
    SShared* S = reinterpret_cast<SShared*>(base + (size_t)NS * SB);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, G = p.G;

    if (threadIdx.x == 0) {
        // full: the TMA lane's arrive + expect_tx and one arrival of the gather group (after
        // its row copies have landed in P2/P3; at once in P0/P1)
        for (int i = 0; i < NS; ++i) { ub_init(&S->full[i], 2); ub_init(&S->empty[i], 1); }
        for (int i = 0; i < 2; ++i) { ub_init(&S->tfull[i], 1); ub_init(&S->tempty[i], 4); }
        ub_init(&S->done, 1);
        S->abort = 0;
        S->flagU = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s32(&S->tmem)),
                     "r"(p.tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem;
    const int Nmax = p.N2;

    if (warp == 0) {
        // =============================================================== TMA producer
        if (lane == 0) {
            int st = 0, ph = 0;
            uint32_t issued = 0, last_ph = 0;
            struct Pend { int st, x; };
            Pend pend[kSMaxStages];
            bool ok = true;
            for (int l = 0; l < p.L && ok; ++l) {
                for (int mode = 0; mode < 4 && ok; ++mode) {
                    int U = 0;
                    if (mode >= 2) {
                        U = wait_U(p, S, l);
                        if (U < 0) { ok = false; break; }
                    }
                    const SPlan q = splan(p, mode, U);
                    // activation tile: x_l (P0, P2), hsplit (P1), asplit (P3), and the grid
                    // barrier after which it is complete
                    const CUtensorMap* bmap = (mode == 0 || mode == 2) ? &p.tmX[x_map(l)] : (mode == 1 ? &p.tmH : &p.tmA);
                    const CUtensorMap* amap = mode == 0 ? &p.tmWp1[l] : &p.tmWp2[l];
                    // (P2 waits for x_l too: a CTA with no P0 tile has not waited for it yet)
                    uint32_t dep = 0;
                    if ((mode == 0 || mode == 2) && l > 0) dep = gb_target(p, l - 1, kSBarriers - 1);
                    if (mode == 1) dep = gb_target(p, l, 0);
                    if (mode == 3) dep = gb_target(p, l, 2);
                    bool met = dep == 0 || ld_acq(p.bar) >= dep;
                    if (met && dep) fence_async_global();
                    int npend = 0;
                    auto flush = [&]() {
                        fence_async_global();
                        for (int i = 0; i < npend; ++i)
                            tma_2d(base + (size_t)pend[i].st * SB + 16384, bmap, pend[i].x, 0, &S->full[pend[i].st]);
                        npend = 0;
                    };
                    const uint32_t bbytes = (uint32_t)q.N * 128u;
                    for (int u = c; u < q.units && ok; u += G) {
                        const int tile = u / q.splits, sp = u % q.splits;
                        const int kb0 = kb_lo(q, sp), kb1 = kb_lo(q, sp + 1);
                        for (int kb = kb0; kb < kb1; ++kb) {
                            if (!mb_wait(p, S, &S->empty[st], ph ^ 1)) { ok = false; break; }
                            char* sa = base + (size_t)st * SB;
                            if (mode <= 1) {
                                ub_expect(&S->full[st], 16384u + bbytes);
                                tma_2d(sa, amap, kb * kSBK, tile * kSBM, &S->full[st]);
                            } else {
                                ub_expect(&S->full[st], bbytes);     // the gather group copies the A rows
                            }
                            if (!met) {
                                met = ld_acq(p.bar) >= dep;
                                if (met) {
                                    if (l < p.L && mode == 1) STRACE(9);
                                    if (l < p.L && mode == 3) STRACE(10);
                                    flush();
                                }
                            }
                            if (met) {
                                tma_2d(sa + 16384, bmap, kb * kSBK, 0, &S->full[st]);
                            } else {
                                pend[npend++] = {st, kb * kSBK};
                                if (npend == NS) {
                                    if (!gb_wait(p, S, dep)) { ok = false; break; }
                                    met = true;
                                    flush();
                                }
                            }
                            issued |= 1u << st;
                            last_ph = (last_ph & ~(1u << st)) | ((uint32_t)ph << st);
                            if (++st == NS) { st = 0; ph ^= 1; }
                        }
                    }
                    if (ok && npend) {
                        if (!gb_wait(p, S, dep)) ok = false;
                        else flush();
                    }
                }
            }
            // on abort: wait (bounded) for the last fill of every stage this lane issued into
            if (!ok || aborted(p, S)) {
                for (int s = 0; s < NS; ++s) {
                    if (!((issued >> s) & 1u)) continue;
                    const unsigned long long t0 = now_ns();
                    while (!ub_try(&S->full[s], (last_ph >> s) & 1u) && now_ns() - t0 < kSDrainNs) {}
                }
                const unsigned long long t0 = now_ns();
                while (now_ns() - t0 < 200000ull) {}
            }
        }
    } else if (warp >= 6) {
        // =============================================================== row gathers (P2, P3)
        // P2: the tile's 128 table rows of W1, 128 bytes of each per K block (eight lanes per
        //     row), at r*128 with the 128-byte swizzle (K-major image).
        // P3: K block kb = table rows kb*64..+63 of W2T, 256 bytes of each (this tile's 128
        //     output columns: two 64-column blocks 8 KB apart, row r at r*128, swizzled:
        //     the MN-major image).  Sixteen lanes per row.
        // Each thread commits one cp.async group per stage and keeps up to kSLag - 1 groups in
        // flight; once the oldest has landed it fences it into the async proxy, and after a
        // group barrier one thread gives the group's arrival on that stage's full barrier.
        const int t = threadIdx.x - 6 * 32;
        // a stage's arrival comes lag - 1 fills after its copies; more groups in flight measured
        // slower for these scattered row pieces (the rate falls as requests queue up)
        const int lag = kSLag;
        int st = 0, ph = 0, nlag = 0, nb = 0;
        int lag_st[kSMaxStages];
        bool ok = true;
        // thread 0 decides, the group follows (parity-buffered, so a fast thread's next
        // decision cannot overwrite one a slow thread has not read yet)
        auto group_ok = [&](bool v0) -> bool {
            const int k = nb++ & 1;
            if (t == 0) S->gok[k] = v0;
            gather_sync();
            return S->gok[k] != 0;
        };
        auto settle_all = [&]() {
            cp_async_wait<0>();
            fence_async_smem();
            gather_sync();
            if (t == 0)
                for (int i = 0; i < nlag; ++i) ub_arrive(&S->full[lag_st[i]]);
            nlag = 0;
        };
        const int32_t* tab = p.ptab + (size_t)c * p.n;       // this CTA's copy of the table
        for (int l = 0; l < p.L && ok; ++l) {
            const char* W1 = reinterpret_cast<const char*>(p.layer[l].W1);
            const char* W2 = reinterpret_cast<const char*>(p.layer[l].W2T);
            for (int mode = 0; mode < 4 && ok; ++mode) {
                int U = 0;
                if (mode >= 2) {
                    // U is published once this CTA's copy of the table is written
                    bool g = true;
                    if (t == 0) {
                        g = wait_U(p, S, l) >= 0;
                        __threadfence_block();
                    }
                    if (!group_ok(g)) { ok = false; break; }
                    U = *(volatile int*)&S->U[l & 1];
                }
                const SPlan q = splan(p, mode, U);
                if (mode <= 1) {
                    // TMA tiles only: thread 0 gives the group's arrival as each stage frees up;
                    // every thread keeps the ring position in step
                    bool g = true;
                    for (int u = c; u < q.units; u += G) {
                        const int sp = u % q.splits;
                        const int nf = kb_lo(q, sp + 1) - kb_lo(q, sp);
                        for (int f = 0; f < nf; ++f) {
                            if (t == 0 && g) {
                                g = mb_wait(p, S, &S->empty[st], ph ^ 1);
                                if (g) ub_arrive(&S->full[st]);
                            }
                            if (++st == NS) { st = 0; ph ^= 1; }
                        }
                    }
                    if (!group_ok(g)) { ok = false; break; }
                    continue;
                }
                for (int u = c; u < q.units && ok; u += G) {
                    const int tile = u / q.splits, sp = u % q.splits;
                    const int kb0 = kb_lo(q, sp), kb1 = kb_lo(q, sp + 1);
                    const char* rows[8];
                    const int c2 = t & 7;                               // P2: 16-byte chunk of the row piece
                    const int ch = t & 15, mb = ch >> 3, c3 = ch & 7;   // P3
                    auto fc2_rows = [&](int kb) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int r = kb * kSBK + i * 8 + (t >> 4);
                            int j = r < U ? __ldcg(tab + r) : 0;
                            j = (unsigned)j < (unsigned)p.n ? j : 0;
                            rows[i] = W2 + (size_t)j * p.d * 2;
                        }
                    };
                    if (mode == 2) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int r = tile * kSBM + i * 16 + (t >> 3);
                            int j = __ldcg(tab + (r < U ? r : 0));
                            j = (unsigned)j < (unsigned)p.n ? j : 0;
                            rows[i] = W1 + (size_t)j * p.d * 2 + c2 * 16;
                        }
                    } else if (kb0 < kb1) {
                        fc2_rows(kb0);
                    }
                    const size_t col3 = ((size_t)tile * kSBM + mb * 64 + c3 * 8) * 2;
                    for (int kb = kb0; kb < kb1; ++kb) {
                        if (nlag == lag - 1) {
                            cp_async_wait_n(lag - 2);          // the oldest pending group has landed
                            fence_async_smem();
                        }
                        bool g = true;
                        if (t == 0) g = mb_wait(p, S, &S->empty[st], ph ^ 1);
                        const bool go = group_ok(g);
                        if (nlag == lag - 1) {
                            if (t == 0) ub_arrive(&S->full[lag_st[0]]);
                            for (int i = 0; i + 1 < nlag; ++i) lag_st[i] = lag_st[i + 1];
                            --nlag;
                        }
                        if (!go) { ok = false; break; }
                        char* sa = base + (size_t)st * SB;
                        if (mode == 2) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int r = i * 16 + (t >> 3);
                                cp_async16(sa + r * 128 + ((c2 ^ (r & 7)) << 4), rows[i] + (size_t)kb * kSBK * 2);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int r = i * 8 + (t >> 4);
                                cp_async16(sa + mb * 8192 + r * 128 + ((c3 ^ (r & 7)) << 4), rows[i] + col3);
                            }
                            if (kb + 1 < kb1) fc2_rows(kb + 1);
                        }
                        cp_async_commit();
                        lag_st[nlag++] = st;
                        if (++st == NS) { st = 0; ph ^= 1; }
                    }
                }
                if (mode == 3 || !ok) settle_all();
            }
        }
        if (nlag) settle_all();
    } else if (warp == 1) {
        // =============================================================== MMA issuer
        if (lane == 0) {
            int st = 0, ph = 0, ab = 0, aph = 0;
            bool any = false, ok = true;
            for (int l = 0; l < p.L && ok; ++l) {
                for (int mode = 0; mode < 4 && ok; ++mode) {
                    int U = 0;
                    if (mode >= 2) {
                        U = wait_U(p, S, l);
                        if (U < 0) { ok = false; break; }
                    }
                    const SPlan q = splan(p, mode, U);
                    const uint32_t idesc = (1u << 4) | ((uint32_t)p.dtype << 7) | ((uint32_t)p.dtype << 10) |
                                           ((mode == 3 ? 1u : 0u) << 15) | ((uint32_t)(q.N >> 3) << 17) |
                                           ((uint32_t)(kSBM >> 4) << 24);
                    bool first = true;
                    for (int u = c; u < q.units && ok; u += G) {
                        const int sp = u % q.splits;
                        const int kb0 = kb_lo(q, sp), kb1 = kb_lo(q, sp + 1);
                        if (kb1 == kb0) continue;
                        if (!mb_wait(p, S, &S->tempty[ab], aph ^ 1)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t d_tmem = tmem + (uint32_t)(ab * Nmax);
                        for (int kb = kb0; kb < kb1; ++kb) {
                            if (!mb_wait(p, S, &S->full[st], ph)) { ok = false; break; }
                            tc_fence_after();
                            if (first && mode >= 2) { STRACE(mode == 2 ? 11 : 12); first = false; }
                            const uint32_t sa = s32(base + (size_t)st * SB), sb = sa + 16384u;
#pragma unroll
                            for (int k = 0; k < kSBK / 16; ++k) {
                                const uint64_t adesc = mode == 3 ? sdesc(sa + k * 2048u, 512u, 64u) : sdesc(sa + k * 32u, 1u, 64u);
                                const uint64_t bdesc = sdesc(sb + k * 32u, 1u, 64u);
                                umma(d_tmem, adesc, bdesc, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
                            }
                            ucommit(&S->empty[st]);
                            any = true;
                            if (++st == NS) { st = 0; ph ^= 1; }
                        }
                        if (!ok) break;
                        ucommit(&S->tfull[ab]);
                        if (++ab == 2) { ab = 0; aph ^= 1; }
                    }
                }
            }
            if (any) {
                ucommit(&S->done);
                const unsigned long long t0 = now_ns();
                while (!ub_try(&S->done, 0) && now_ns() - t0 < kUWaitNs) {}
            }
        }
    } else {
        // =============================================================== epilogue (warps 2..5)
        const int quad = warp & 3;
        const int lane_row = quad * 32 + lane;
        const int et = threadIdx.x - 64;
        int ab = 0, aph = 0, nb = 0;
        bool ok = true;
        // thread 0 decides, the group follows (parity-buffered like the gather group's)
        auto group_ok = [&](bool v0) -> bool {
            const int k = nb++ & 1;
            if (et == 0) S->eok[k] = v0;
            epi_sync();
            return S->eok[k] != 0;
        };
        auto group_gb = [&](uint32_t target) -> bool {
            bool g = true;
            if (et == 0) g = gb_wait(p, S, target);
            return group_ok(g);
        };
        // Arrival on grid barrier b of layer l.  The counter is monotonic, so a CTA arrives at
        // a barrier only once it has seen the previous one complete: otherwise a CTA with no
        // work in a phase could arrive twice before a slow CTA arrives once, and the count
        // would pass the earlier barrier's target too soon.
        auto arrive = [&](int l, int b) -> bool {
            const bool seen = (l == 0 && b == 0) ||
                              group_gb(b > 0 ? gb_target(p, l, b - 1) : gb_target(p, l - 1, kSBarriers - 1));
            __threadfence();
            fence_async_global();
            epi_sync();
            if (seen && et == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.bar) : "memory");
            return seen;
        };
        for (int l = 0; l < p.L && ok; ++l) {
            if (et == 0) STRACE(0);
            // x_l complete (written by every CTA's chaining of layer l - 1)
            if (l > 0 && !group_gb(gb_target(p, l - 1, kSBarriers - 1))) { ok = false; break; }
            const T* xl = reinterpret_cast<const T*>(x_ptr(p, l));
            const SLayer& Ly = p.layer[l];
            const bool last_layer = l == p.L - 1;
            int U = 0;
            for (int mode = 0; mode < 4 && ok; ++mode) {
                if (mode == 2) {
                    // ---- C: the neuron table from the mask words: every CTA computes the prefix,
                    //      expands the whole table into its own copy and writes its slice of
                    //      words into the layer's table (the caller's copy)
                    if (!group_gb(gb_target(p, l, 1))) { ok = false; break; }
                    const int W = p.n >> 5;
                    const int per = (W + 127) / 128;
                    const int w0 = min(W, et * per), w1 = min(W, w0 + per);
                    int local = 0;
                    for (int w = w0; w < w1; ++w) local += __popc(__ldcg(p.mask + w));
                    S->scan[et] = local;
                    epi_sync();
                    if (et == 0) {
                        int run = 0;
                        for (int i = 0; i < 128; ++i) { const int v = S->scan[i]; S->scan[i] = run; run += v; }
                        S->U[l & 1] = run;
                    }
                    epi_sync();
                    U = S->U[l & 1];
                    const int sw0 = (int)((long long)W * c / G), sw1 = (int)((long long)W * (c + 1) / G);
                    int32_t* own = p.ptab + (size_t)c * p.n;
                    int pos = S->scan[et];
                    for (int w = w0; w < w1; ++w) {
                        uint32_t bits = __ldcg(p.mask + w);
                        const bool mine = w >= sw0 && w < sw1;
                        while (bits) {
                            const int b = __ffs(bits) - 1;
                            bits &= bits - 1;
                            own[pos] = w * 32 + b;
                            if (mine) Ly.idx[pos] = w * 32 + b;
                            ++pos;
                        }
                    }
                    __threadfence_block();
                    epi_sync();
                    if (et == 0) {
                        if (c == 0 && p.counts) p.counts[l] = U;
                        __threadfence_block();
                        *(volatile int*)&S->flagU = l + 1;     // TMA, MMA and gathers may run P2, P3
                        STRACE(3);
                    }
                }
                const SPlan q = splan(p, mode, U);
                const bool pair = mode == 1 || mode == 3;
                const int half = pair ? p.N1 : q.N;
                for (int u = c; u < q.units && ok; u += G) {
                    const int tile = u / q.splits, sp = u % q.splits;
                    const int kb0 = kb_lo(q, sp), kb1 = kb_lo(q, sp + 1);
                    const bool has = kb1 > kb0;
                    uint32_t taddr = 0;
                    if (has) {
                        bool g = true;
                        if (et == 0) g = mb_wait(p, S, &S->tfull[ab], aph);
                        if (!group_ok(g)) { ok = false; break; }
                        tc_fence_after();
                        taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(ab * Nmax);
                    }
                    const int r = tile * kSBM + lane_row;
                    // final values of 16 columns (c0..c0+15 of each half) of this thread's D row
                    auto finish = [&](int c0, const float* hi, const float* lo, bool& anyb, float* sq) {
                        if (mode == 0) {
                            if (r < p.H) {
                                const float bias = ldf<T>(Ly.bp1, r);
                                T* hs = reinterpret_cast<T*>(p.hsplit);
                                for (int i = 0; i < 16 && c0 + i < p.B; ++i) {
                                    const int t = c0 + i;
                                    const float h = fmaxf(hi[i] + bias, 0.f);
                                    const T h1 = DT<T>::r(h);
                                    const T h2 = DT<T>::r(h - DT<T>::f(h1));
                                    hs[(size_t)t * p.H + r] = h1;
                                    hs[(size_t)(p.N1 + t) * p.H + r] = h2;
                                }
                            }
                        } else if (mode == 1) {
                            if (r < p.n) {
                                const float bias = ldf<T>(Ly.bp2, r);
                                for (int i = 0; i < 16 && c0 + i < p.B; ++i) anyb |= (hi[i] + lo[i] + bias) > 0.f;
                            }
                        } else if (mode == 2) {
                            if (r < q.tiles * kSBM && r < p.n) {
                                const int j = r < U ? __ldcg(p.ptab + (size_t)c * p.n + r) : -1;
                                const bool live = (unsigned)j < (unsigned)p.n;
                                const float bias = live ? ldf<T>(Ly.b1, j) : 0.f;
                                T* as = reinterpret_cast<T*>(p.asplit);
                                for (int i = 0; i < 16 && c0 + i < p.B; ++i) {
                                    const int t = c0 + i;
                                    const float a = live ? fmaxf(hi[i] + bias, 0.f) : 0.f;
                                    const T a1 = DT<T>::r(a);
                                    const T a2 = DT<T>::r(a - DT<T>::f(a1));
                                    as[(size_t)t * p.n + r] = a1;
                                    as[(size_t)(p.N1 + t) * p.n + r] = a2;
                                }
                            }
                        } else {
                            // y = D + b2, u = x_l + y (and y itself for the last layer); u^2 per token
                            const float bias = ldf<T>(Ly.b2, r);
                            for (int i = 0; i < 16; ++i) {
                                const int t = c0 + i;
                                float v = 0.f;
                                if (t < p.B) {
                                    const float yv = hi[i] + lo[i] + bias;
                                    const float uv = DT<T>::f(xl[(size_t)t * p.d + r]) + yv;
                                    __stcg(p.u + (size_t)t * p.d + r, uv);
                                    if (last_layer) p.y[(size_t)t * p.d + r] = yv;
                                    v = uv * uv;
                                }
                                sq[i] = v;
                            }
                        }
                    };
                    // per token: the sum over the tile's 128 rows of u^2, in a fixed order
                    auto tile_ss = [&](int c0, const float* sq) {
                        float w[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) w[i] = warp_sum(sq[i]);
                        if (lane == 0)
#pragma unroll
                            for (int i = 0; i < 16; ++i) S->red[quad][i] = w[i];
                        epi_sync();
                        if (et < 16 && c0 + et < p.B) {
                            const float s = (S->red[0][et] + S->red[1][et]) + (S->red[2][et] + S->red[3][et]);
                            __stcg(p.ss + (size_t)tile * p.B + c0 + et, s);
                        }
                        epi_sync();
                    };
                    if (q.splits == 1) {
                        bool anyb = false;
                        for (int c0 = 0; c0 < half; c0 += 16) {
                            float hi[16], lo[16], sq[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) hi[i] = lo[i] = 0.f;
                            if (has) {
                                tmem_ld16(taddr + c0, hi);
                                if (pair) tmem_ld16(taddr + half + c0, lo);
                                tmem_wait_ld();
                            }
                            finish(c0, hi, lo, anyb, sq);
                            if (mode == 3) tile_ss(c0, sq);
                        }
                        if (mode == 1) {
                            const uint32_t bits = __ballot_sync(0xffffffffu, anyb);
                            const int word = (tile * kSBM + (lane_row & ~31)) >> 5;
                            if (lane == 0 && word < (p.n >> 5)) p.mask[word] = bits;
                        }
                    } else {
                        float* mine = p.partial + ((size_t)u * kSBM + lane_row) * q.N;
                        for (int c0 = 0; c0 < q.N; c0 += 16) {
                            float v[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) v[i] = 0.f;
                            if (has) {
                                tmem_ld16(taddr + c0, v);
                                tmem_wait_ld();
                            }
#pragma unroll
                            for (int i = 0; i < 16; i += 4)
                                __stcg(reinterpret_cast<float4*>(mine + c0 + i), make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]));
                        }
                    }
                    if (has) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ub_arrive(&S->tempty[ab]);
                        if (++ab == 2) { ab = 0; aph ^= 1; }
                    }
                    if (q.splits == 1) continue;
                    // the last CTA to finish a split of this tile sums the splits in split order
                    __threadfence();
                    epi_sync();
                    if (et == 0) S->last = atomicAdd(&p.tickets[tile], 1u) == (uint32_t)(q.splits - 1);
                    epi_sync();
                    if (S->last) {
                        __threadfence();
                        bool anyb = false;
                        for (int c0 = 0; c0 < half; c0 += 16) {
                            float hi[16], lo[16], sq[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) hi[i] = lo[i] = 0.f;
                            for (int s = 0; s < q.splits; ++s) {
                                const float4* src = reinterpret_cast<const float4*>(
                                    p.partial + ((size_t)(tile * q.splits + s) * kSBM + lane_row) * q.N + c0);
#pragma unroll
                                for (int c4 = 0; c4 < 4; ++c4) {
                                    const float4 a = __ldcg(src + c4);
                                    hi[4 * c4] += a.x; hi[4 * c4 + 1] += a.y; hi[4 * c4 + 2] += a.z; hi[4 * c4 + 3] += a.w;
                                    if (pair) {
                                        const float4 b = __ldcg(src + half / 4 + c4);
                                        lo[4 * c4] += b.x; lo[4 * c4 + 1] += b.y; lo[4 * c4 + 2] += b.z; lo[4 * c4 + 3] += b.w;
                                    }
                                }
                            }
                            finish(c0, hi, lo, anyb, sq);
                            if (mode == 3) tile_ss(c0, sq);
                        }
                        if (et == 0) p.tickets[tile] = 0u;
                    }
                    epi_sync();
                }
                if (!ok) break;
                // P0 -> barrier 0, P1 -> 1, P2 -> 2, P3 -> 3
                if (!arrive(l, mode)) { ok = false; break; }
                if (et == 0) STRACE(mode == 0 ? 1 : (mode == 1 ? 2 : (mode == 2 ? 4 : 5)));
            }
            if (!ok) break;
            // ---- X: x_{l+1} = round(u / sqrt(mean(u^2) + 1e-6)) for this CTA's slice
            if (!group_gb(gb_target(p, l, 3))) { ok = false; break; }
            const int T_ = p.d / kSBM;
            if (et < p.B) {
                float s = 0.f;
                for (int i = 0; i < T_; ++i) s += __ldcg(p.ss + (size_t)i * p.B + et);
                S->rs[et] = 1.0f / sqrtf(s / (float)p.d + 1e-6f);
            }
            epi_sync();
            T* xo = reinterpret_cast<T*>(last_layer ? p.x_out : p.xbuf[l & 1]);
            const int V = p.B * p.d / 8;
            const int v0 = (int)((long long)V * c / G), v1 = (int)((long long)V * (c + 1) / G);
            for (int v = v0 + et; v < v1; v += 128) {
                const int e = v * 8, t = e / p.d;
                const float4* up = reinterpret_cast<const float4*>(p.u + e);
                const float4 a = __ldcg(up), b = __ldcg(up + 1);
                const float rs = S->rs[t];
                const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                T o[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) o[k] = DT<T>::r(f[k] * rs);
                *reinterpret_cast<uint4*>(xo + e) = *reinterpret_cast<const uint4*>(o);
            }
            if (!arrive(l, 4)) { ok = false; break; }
            if (et == 0) STRACE(6);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols));
    }
}

#undef STRACE

size_t ustack_smem(int stages, int stage_bytes) {
    return (size_t)stages * stage_bytes + sizeof(SShared) + 1024;
}

void ustack_geometry(int B, int& N1, int& N2, int& stages, int& stage_bytes, int& tmem_cols) {
    N1 = round16(B);
    N2 = 2 * N1;
    stage_bytes = 16384 + N2 * 128;
    stages = std::min(kSMaxStages, (int)((220 * 1024 - sizeof(SShared) - 1024) / stage_bytes));
    tmem_cols = 32;
    while (tmem_cols < 2 * N2) tmem_cols *= 2;
}

// spffn_set_union_stack: 0 per-layer launches, 1 whole stack for 3 <= B <= 128, 2 (default)
// the faster of the two on the measured shapes, which is per-layer at every batch: the
// per-layer tensor-core kernels, chained by programmatic dependent launch, measured faster at
// B = 3, 4, 8 (OPT-13B shape: 2.40 / 2.44 / 2.52 vs 3.14 / 3.20 / 3.31 ms per step), B = 16
// (2.63 vs 3.97 ms) and B = 32 (OPT-66B shape: 6.57 vs 9.83 ms)
int g_ustack_mode = 2;

}  // namespace

void set_ustack_mode(int mode) { g_ustack_mode = mode; }
int ustack_mode() { return g_ustack_mode; }

bool ustack_supported(spffn_ctx* const* layers, int L, int B)
{
    if (g_ustack_mode != 1) return false;
    // batches below 16 pad the MMA's N to 16 columns: idle tensor-core lanes, the same bytes
    if (L < 1 || L > kSMaxLayers || B < kUStackMinBatch || B > 128) return false;
    const spffn_ctx& c0 = *layers[0];
    if (c0.lay.uss == 0 || c0.lay.utab == 0 || c0.num_sms > kMaxUnionCtas || c0.lay.S != c0.num_sms ||
        encoder() == nullptr)
        return false;
    for (int l = 0; l < L; ++l) {
        const spffn_ctx& c = *layers[l];
        if (B > c.cfg.max_batch || c.cfg.d % 128 != 0 || c.lay.upartial == 0 || c.lay.uss == 0) return false;
        if (c.cfg.d != c0.cfg.d || c.cfg.n != c0.cfg.n || c.cfg.H != c0.cfg.H || c.cfg.dtype != c0.cfg.dtype)
            return false;
    }
    int N1, N2, stages, sb, tc;
    ustack_geometry(B, N1, N2, stages, sb, tc);
    return stages >= kSLag && ustack_smem(stages, sb) <= 227 * 1024;
}

cudaError_t launch_ustack(spffn_ctx* const* layers, int L, const void* x_in, int B, void* x_out, float* y,
                          int32_t* counts, cudaStream_t st)
{
    const spffn_ctx& c0 = *layers[0];
    const spffn_config& g = c0.cfg;
    SParams* p = new (std::nothrow) SParams;   // 20+ KB: keep it off the caller's stack
    if (!p) return cudaErrorMemoryAllocation;
    memset(p, 0, sizeof(*p));
    ustack_geometry(B, p->N1, p->N2, p->stages, p->stage_bytes, p->tmem_cols);
    p->L = L; p->B = B; p->d = g.d; p->n = g.n; p->H = g.H; p->G = c0.num_sms; p->dtype = g.dtype;
    p->x_in = x_in;
    p->xbuf[0] = c0.xbuf(0);
    p->xbuf[1] = c0.xbuf(1);
    p->x_out = x_out;
    p->y = y;
    p->counts = counts;
    p->hsplit = c0.hsplit();
    p->asplit = c0.asplit();
    p->mask = c0.mask();
    p->partial = c0.upartial();
    p->tickets = c0.utickets();
    p->u = c0.ybuf();
    p->ss = c0.uss();
    p->ptab = c0.utab();
    Ctl* ctl = c0.ctl();
    p->bar = &ctl->barrier[2];
    p->abort = &ctl->barrier[3];
    p->err = &ctl->err;
    p->wait_ns = wait_test_ns();
    p->bar_extra = wait_test_bar_extra();
    p->trace = static_cast<unsigned long long*>(trace_buffer((size_t)c0.num_sms * L * kSTraceMarks * 8));
    bool ok = make_map(&p->tmX[0], x_in, g.dtype, B, g.d, p->N1) &&
              make_map(&p->tmX[1], c0.xbuf(0), g.dtype, B, g.d, p->N1) &&
              make_map(&p->tmX[2], c0.xbuf(1), g.dtype, B, g.d, p->N1) &&
              make_map(&p->tmH, c0.hsplit(), g.dtype, p->N2, g.H, p->N2) &&
              make_map(&p->tmA, c0.asplit(), g.dtype, p->N2, g.n, p->N2);
    for (int l = 0; l < L && ok; ++l) {
        const spffn_ctx& c = *layers[l];
        ok = make_map(&p->tmWp1[l], c.w.Wp1, g.dtype, g.H, g.d, kSBM) &&
             make_map(&p->tmWp2[l], c.w.Wp2, g.dtype, g.n, g.H, kSBM);
        p->layer[l] = SLayer{c.w.W1, c.w.b1, c.w.W2T, c.w.b2, c.w.bp1, c.w.bp2, c.idx()};
    }
    if (!ok) { delete p; return cudaErrorInvalidValue; }
    const size_t smem = ustack_smem(p->stages, p->stage_bytes);
    cudaError_t e;
    auto kern = g.dtype == SPFFN_BF16 ? k_ustack<__nv_bfloat16> : k_ustack<__half>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaMemsetAsync(&ctl->barrier[2], 0, 2 * sizeof(uint32_t), st);
    if (e == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(p->G);
        cfg.blockDim = dim3(kSThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, *p);
    }
    delete p;
    return e;
}

}  // namespace spffn
