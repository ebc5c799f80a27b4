// Union-mask tensor-core path for batches of 3..256 tokens (below 16 the MMA's N is padded to 16).
//
// With B tokens the union of the per-token neuron sets is a dense contraction
// over the gathered rows (each weight byte feeds B products), so every GEMM of
// the layer runs on the 5th-generation tensor cores:
//
//   mode 0  predictor-1   D[H x B]    = Wp1[H x d]        . X[B x d]^T          split-K
//   mode 1  predictor-2   D[n x 2Gt]  = Wp2[n x H]        . hsplit_g[2Gt x H]^T -> mask words;
//                         the CTA that finishes last compacts the mask into the table
//   mode 2  FC1 (union)   D[U x B]    = W1[table][U x d]  . X[B x d]^T          split-K
//   mode 3  FC2 (union)   D[d x 2Gt]  = W2T[table]^T      . asplit_g[2Gt x U]^T split-K
//
// fp32 activations (h, a) enter the 16-bit MMA as a hi/lo pair of the storage
// dtype (v ~= hi + lo, hi = round(v), lo = round(v - hi)); the epilogue adds the
// two column halves of D.  X is already in the storage dtype (exact).  Modes 1
// and 3 run once per token group g of Gt <= 128 tokens (N = 2 Gt <= 256).
//
// One persistent CTA per SM:
// - warp 0 issues TMA loads into a ring of 4..6 stages: 2-D tiles for the
//   contiguous operands (never multicast);
// - warps 6..13 gather the table rows of FC1 (K-major, 128-byte pieces) and of
//   FC2 (MN-major, 256-byte pieces) with coalesced 16-byte cp.async into the
//   128-byte swizzled image a TMA tile would leave.  Each thread fences its
//   landed copies into the async proxy before it arrives.  For both patterns
//   this moves rows about 1.7-2x faster than TMA tile::gather4;
// - warp 1 issues tcgen05.mma into a double-buffered TMEM accumulator;
// - warps 2..5 read TMEM (tcgen05.ld), 16 columns at a time, and run the epilogue.
// Split-K partials are summed in fixed split order, so results are deterministic:
// once all splits of a tile have published (an arrival counter, a bounded wait),
// each split's CTA reduces its own share of the tile's rows, so no single CTA
// carries the whole reduction as a tail.
#include <cuda.h>
#include <algorithm>
#include <cstring>
#include "spffn_internal.cuh"
#include "spffn_umma.cuh"
#include "spffn_union.cuh"
#include "spffn_fused.cuh"

namespace spffn {
namespace {
using namespace um;

constexpr int kUThreads = 448;       // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue, 6..13 row gathers
constexpr int kGatherThreads = 256;  // eight gather warps: the gather rate grows with the warps issuing
constexpr int kBM = 128;             // D rows per tile
constexpr int kBK = 64;              // K per stage: one 128-byte swizzle row of 16-bit elements
constexpr int kMaxStages = 6;       // stage = A tile 16 KB + B tile N x 128 B (N <= 256)
constexpr int kMaxN = 256;           // MMA N per launch; TMEM holds two accumulators of N columns
constexpr int kGroup = 128;          // tokens per group of the split-activation modes (1, 3)
constexpr int kMaxCluster = 8;        // portable thread-block cluster size
constexpr int kTicketCompact = kUnionTickets - 1;   // mode 1: CTAs done with their mask words
// Split-K hand-off through global memory, per tile (a tile with splits > 1 has index < the
// CTA count <= kMaxUnionCtas): tickets[kTicketArrive + tile] counts split arrivals and never
// resets; tickets[kTicketBase + tile] holds its value before the current call's arrivals.
constexpr int kTicketArrive = 1024;
constexpr int kTicketBase = 1536;
constexpr unsigned long long kUDrainNs = 20000000ull;   // per stage, abort path only
// Time stamps of one launch (tracing aid, per CTA): 0 set up, 1 TMA lane past the wait for
// the previous kernel, 2 first stage consumed by the MMA, 3 last MMA issued, 4 last
// accumulator read, 5 epilogue done (split reduction included), 6 gathers issued, 7 exit.
constexpr int kUTraceMarks = 8;
#define UTRACE(mark)                                                                     \
    do {                                                                                 \
        if (p.trace) p.trace[(size_t)blockIdx.x * kUTraceMarks + (mark)] = now_ns();     \
    } while (0)

struct alignas(64) UParams {
    CUtensorMap tmA;      // modes 0, 1: the weight operand (2-D tiles)
    CUtensorMap tmB;      // the activation operand (2-D tiles)
    int mode, B, N, dtype;
    int M;                // D rows when known on the host (modes 0, 1, 3)
    int K;                // contraction length when known on the host (modes 0, 1, 2)
    int n, d, H, G;
    int splits_fixed;     // mode 0
    int stages, stage_bytes, tmem_cols;
    int Gs;               // modes 0, 2: token-group size of the split buffer written (hsplit, asplit)
    int Gt, Bt, t_base, b_row0, mask_or;   // modes 1, 3: this group's size (hi/lo column offset),
                                           // valid tokens, first token, first B-operand row, OR mask
    const int32_t* count; // modes 2, 3: table length U (device)
    const int32_t* idx;   // modes 2, 3: neuron table
    const void* W;        // mode 2: W1, mode 3: W2T, rows gathered by the table
    const void* bias;     // bp1, bp2, b1 (by neuron), b2
    float* partial;       // [units][kBM][N]
    uint32_t* tickets;    // [tiles]
    void* out_split;      // mode 0: hsplit, mode 2: asplit: [groups][2][Gs][H or n] hi/lo pairs
    float* out_f32;       // mode 0: h [B][H] (may be null); mode 3: y [B][d]
    uint32_t* mask;       // mode 1
    int32_t* cidx;        // mode 1, last token group: the CTA finishing last writes the neuron table
    int32_t* ccount;      //   here, its length here and (if not null) in ccount2
    int32_t* ccount2;
    int32_t* tpriv;       // mode 2, not null: the CTAs rank the mask words themselves, each into its own
                          //   table copy tpriv[CTA][n], and write the table to cidx and its length to
                          //   ccount (and ccount2)
    uint32_t* err;
    unsigned long long* trace;   // null, or this launch's [CTA][kUTraceMarks] time stamps
    int cluster;          // > 1: the splits of a tile form one thread-block cluster of this size
    int red_off, rpo;     //   and reduce through distributed shared memory: the reduction buffer's
                          //   offset in shared memory, and tile rows owned per CTA of the cluster
};

// Work decomposition shared by all three roles (same answer in every thread).
struct Plan {
    int tiles, splits, kblocks, M, K;
    const int32_t* tab;   // modes 2, 3: the neuron table the rows come from
};
// Uown >= 0: mode 2's table length as this CTA ranked it from the mask words
__device__ __forceinline__ Plan make_plan(const UParams& p, int Uown = -1) {
    Plan q;
    q.tab = p.tpriv ? p.tpriv + (size_t)blockIdx.x * p.n : p.idx;
    if (p.mode == 2) {
        int U = Uown >= 0 ? Uown : *reinterpret_cast<const volatile int32_t*>(p.count);
        U = U < 0 ? 0 : (U > p.n ? p.n : U);
        q.M = U;
        q.K = p.K;
    } else if (p.mode == 3) {
        int U = *reinterpret_cast<const volatile int32_t*>(p.count);
        U = U < 0 ? 0 : (U > p.n ? p.n : U);
        q.M = p.M;
        q.K = U;
    } else {
        q.M = p.M;
        q.K = p.K;
    }
    q.tiles = (q.M + kBM - 1) / kBM;
    q.kblocks = (q.K + kBK - 1) / kBK;
    if (p.mode == 0) {
        q.splits = p.splits_fixed;
    } else if (p.mode == 1) {
        q.splits = 1;
    } else {
        const int s = q.tiles > 0 ? p.G / q.tiles : 1;
        q.splits = max(1, min(s, q.kblocks));
    }
    if (q.kblocks > 0 && q.splits > q.kblocks) q.splits = q.kblocks;
    if (p.cluster > 1) q.splits = p.cluster;   // one CTA per split (an empty K range adds zeros)
    return q;
}

template <typename T>
__device__ __forceinline__ float tof(const void* base, int i) {
    return DT<T>::f(reinterpret_cast<const T*>(base)[i]);
}

// Final epilogue for one D row (this thread's TMEM lane) and 16 columns c0..c0+15
// of each half.  Modes 0 and 2 keep one column per token; modes 1 and 3 hold each
// token's hi and lo halves Gt columns apart.  Mode 1 ORs its union decision into *any.
// Per output row of a tile: its bias and whether it is written (0 no, 1 as zeros: a
// mode-2 row past U or with an out-of-range table entry, 2 from the accumulators).
// Loaded before the accumulators are ready, off the epilogue's critical path.
template <typename T>
__device__ __forceinline__ int row_pre(const UParams& p, const Plan& q, int tile, int lane_row, float& bias) {
    const int r = tile * kBM + lane_row;
    bias = 0.f;
    if (p.mode == 2) {
        if (r >= p.n) return 0;
        const int j = r < q.M ? q.tab[r] : -1;
        if ((unsigned)j >= (unsigned)p.n) return 1;
        bias = tof<T>(p.bias, j);
        return 2;
    }
    const int lim = p.mode == 0 ? p.H : (p.mode == 1 ? p.n : p.d);
    if (r >= lim) return 0;
    if (p.bias) bias = tof<T>(p.bias, r);
    return 2;
}

// The epilogue of nc accumulator columns c0.. of one tile row (hi, and in modes 1 and 3
// the matching lo half): state and bias from row_pre.
template <typename T>
__device__ void finish_chunk(const UParams& p, int tile, int lane_row, int c0, const float* hi, const float* lo,
                             bool* any, int nc, int state, float bias)
{
    if (state == 0) return;
    const int r = tile * kBM + lane_row;
    if (p.mode == 0) {                      // h = ReLU(D + bp1) -> fp32 and its hi/lo pair
        T* hs = reinterpret_cast<T*>(p.out_split);
        for (int i = 0; i < nc && c0 + i < p.B; ++i) {
            const int t = c0 + i, g = t / p.Gs, tt = t - g * p.Gs;
            const float h = fmaxf(hi[i] + bias, 0.f);
            const T h1 = DT<T>::r(h);
            const T h2 = DT<T>::r(h - DT<T>::f(h1));
            hs[(size_t)(2 * g * p.Gs + tt) * p.H + r] = h1;
            hs[(size_t)(2 * g * p.Gs + p.Gs + tt) * p.H + r] = h2;
            if (p.out_f32) p.out_f32[(size_t)t * p.H + r] = h;
        }
    } else if (p.mode == 1) {               // union decision over this group's tokens
        for (int i = 0; i < nc && c0 + i < p.Bt; ++i) *any |= (hi[i] + lo[i] + bias) > 0.f;
    } else if (p.mode == 2) {               // a = ReLU(D + b1[j]) for table entry r (zeros past U)
        T* as = reinterpret_cast<T*>(p.out_split);
        for (int i = 0; i < nc && c0 + i < p.B; ++i) {
            const int t = c0 + i, g = t / p.Gs, tt = t - g * p.Gs;
            const float a = state == 2 ? fmaxf(hi[i] + bias, 0.f) : 0.f;
            const T a1 = DT<T>::r(a);
            const T a2 = DT<T>::r(a - DT<T>::f(a1));
            as[(size_t)(2 * g * p.Gs + tt) * p.n + r] = a1;
            as[(size_t)(2 * g * p.Gs + p.Gs + tt) * p.n + r] = a2;
        }
    } else {                                // y[t][c] = D[c][t] + D[c][Gt+t] + b2[c]
        for (int i = 0; i < nc && c0 + i < p.Bt; ++i)
            p.out_f32[(size_t)(p.t_base + c0 + i) * p.d + r] = hi[i] + lo[i] + bias;
    }
}

// Stream compaction of the union mask by all kUThreads threads of one CTA: each thread
// loads its run of up to kCompactWords words at once (one round trip), a block scan of
// the popcounts gives its first slot, and it writes its words' set bits in ascending order.
constexpr int kCompactWords = 8;   // the fused compaction handles n <= kCompactWords * kUThreads * 32

// The block scan shared by the compaction and by FC1's own ranking: thread i loads its run
// of up to kCompactWords mask words (from w0) at once; returns the number of set bits before
// its run in *first and the total over all words.
__device__ uint32_t rank_words(const uint32_t* mask, int words, uint32_t (&wv)[kCompactWords], int& w0,
                               uint32_t* first, uint32_t* wsum)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kUThreads / 32;
    const int per = (words + kUThreads - 1) / kUThreads;
    w0 = min(words, tid * per);
    const int w1 = min(words, w0 + per);
    uint32_t local = 0;
#pragma unroll
    for (int k = 0; k < kCompactWords; ++k) {
        wv[k] = w0 + k < w1 ? __ldcg(mask + w0 + k) : 0u;
        local += __popc(wv[k]);
    }
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint32_t base = 0, total = 0;
#pragma unroll
    for (int k = 0; k < kWarps; ++k) {
        base += k < warp ? wsum[k] : 0u;
        total += wsum[k];
    }
    *first = base + incl - local;
    return total;
}

__device__ void compact_mask_cta(const uint32_t* mask, int words, int32_t* idx, int32_t* count, int32_t* count2,
                                 uint32_t* wsum)
{
    uint32_t wv[kCompactWords];
    int w0;
    uint32_t pos;
    const uint32_t total = rank_words(mask, words, wv, w0, &pos, wsum);
#pragma unroll
    for (int k = 0; k < kCompactWords; ++k) {
        uint32_t bits = wv[k];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            idx[pos++] = (w0 + k) * 32 + b;
        }
    }
    if (threadIdx.x == 0) {
        *count = (int32_t)total;
        if (count2) *count2 = (int32_t)total;
    }
}

template <typename T>
__global__ void __launch_bounds__(kUThreads, 1) k_umma(const __grid_constant__ UParams p)
{
    extern __shared__ __align__(1024) char usm[];
    char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(usm) + 1023) & ~uintptr_t(1023));
    const int kStages = p.stages, kStageBytes = p.stage_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
    uint64_t* empty = full + kMaxStages;
    uint64_t* tfull = empty + kMaxStages;    // [2]
    uint64_t* tempty = tfull + 2;            // [2]
    uint64_t* done = tempty + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(done + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 2);
    int* s_go = reinterpret_cast<int*>(done + 3);      // split-K: every split of the tile is in
    __shared__ uint32_t s_wsum[kUThreads / 32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        // modes 2, 3: the TMA warp's B tile plus one arrival per gathering thread
        const uint32_t fc = (p.mode >= 2) ? 1u + kGatherThreads : 1u;
        for (int i = 0; i < kStages; ++i) { ub_init(&full[i], fc); ub_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { ub_init(&tfull[i], 1); ub_init(&tempty[i], 4); }
        ub_init(done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s32(tmem_slot)),
                     "r"(p.tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) UTRACE(0);
    // Programmatic dependent launch: the next kernel may launch now (its CTAs take an SM as
    // this kernel's CTA there retires).  Everything read from the previous kernel's outputs
    // waits for it: the table length and rows (modes 2, 3) from the start; in modes 0 and 1
    // the TMA lane first issues weight tiles, which do not depend on it.
    pdl_trigger();
    if (p.mode >= 2 || (warp != 0 && warp != 1)) pdl_wait();
    // Mode 2 with its own ranking: every CTA scans the union mask words (left by the logits
    // launch) and keeps the table entries of its own tiles; the CTA holding split 0 of a tile
    // also writes that tile's entries to the shared table, and CTA 0 writes the length.
    uint32_t wv[kCompactWords];
    int w0 = 0, Uown = -1;
    uint32_t rank = 0;                       // set bits before this thread's words
    if (p.mode == 2 && p.tpriv) Uown = (int)rank_words(p.mask, p.n >> 5, wv, w0, &rank, s_wsum);
    const Plan q = make_plan(p, Uown);
    if (Uown >= 0) {
        const int units0 = q.tiles * q.splits, b = blockIdx.x, G = gridDim.x;
        int32_t* own = p.tpriv + (size_t)b * p.n;
        // this CTA's units b, b + G, ..: tile u / splits, ranks [tile kBM, tile kBM + kBM); a
        // thread skips its words outside that window by their popcounts
        for (int u = b; u < units0; u += G) {
            const int t = u / q.splits;
            const bool lead = u % q.splits == 0;
            const uint32_t lo = (uint32_t)t * kBM, hi = min(lo + kBM, (uint32_t)Uown);
            uint32_t r = rank;
#pragma unroll
            for (int k = 0; k < kCompactWords; ++k) {
                const uint32_t nb = __popc(wv[k]);
                if (r + nb <= lo || r >= hi) {
                    r += nb;
                    continue;
                }
                uint32_t bits = wv[k];
                while (bits) {
                    const int j = (w0 + k) * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    if (r >= lo && r < hi) {
                        own[r] = j;
                        if (lead) p.cidx[r] = j;
                    }
                    ++r;
                }
            }
        }
        if (b == 0 && threadIdx.x == 0) {
            *p.ccount = Uown;
            if (p.ccount2) *p.ccount2 = Uown;
        }
        __syncthreads();
    }
    if (p.mode == 2 && !p.tpriv && blockIdx.x == 0 && threadIdx.x == 0) {
        const int U = *p.count;
        if (U < 0 || U > p.n) atomicOr(p.err, ERR_COUNT_CLAMPED);    // clamped by make_plan
    }
    const int units = q.tiles * q.splits;
    const int N = p.N;
    const uint32_t btile_bytes = (uint32_t)N * 128u;

    if (warp == 0) {
        // ------------------------------------------------------------- TMA producer (whole warp)
        // modes 0, 1: A and B tiles (2-D); modes 2, 3: the B tile only (the gather warps copy
        // the A rows of the neuron table)
        int st = 0, ph = 0;
        uint32_t issued = 0, last_ph = 0;    // stages ever filled, parity of each one's last fill
        // modes 0, 1: the first ring's worth of weight tiles goes out before the wait for the
        // previous kernel; their activation tiles follow it
        bool waited = p.mode >= 2;
        int pend_st[kMaxStages], pend_kb[kMaxStages], npend = 0;
        if (waited && lane == 0) UTRACE(1);
        auto release = [&]() {
            if (lane == 0) {
                pdl_wait();
                UTRACE(1);
            }
            __syncwarp();
            waited = true;
            for (int i = 0; i < npend; ++i)
                if (lane == 0) tma_2d(base + pend_st[i] * kStageBytes + 16384, &p.tmB, pend_kb[i] * kBK, p.b_row0,
                                      &full[pend_st[i]]);
            npend = 0;
        };
        for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
            const int tile = u / q.splits, sp = u % q.splits;
            const int kb0 = (int)((long long)sp * q.kblocks / q.splits);
            const int kb1 = (int)((long long)(sp + 1) * q.kblocks / q.splits);
            bool okw = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!waited && npend == kStages) release();     // every stage holds a pending tile
                if (lane == 0) okw = ub_wait(&empty[st], ph ^ 1, abort_flag, p.err);
                okw = __shfl_sync(0xffffffffu, okw, 0);
                if (!okw) break;
                char* sa = base + st * kStageBytes;
                char* sb = sa + 16384;
                if (lane == 0) ub_expect(&full[st], (p.mode >= 2 ? 0u : 16384u) + btile_bytes);
                __syncwarp();
                if (p.mode <= 1) {
                    if (lane == 0) tma_2d(sa, &p.tmA, kb * kBK, tile * kBM, &full[st]);
                }
                if (!waited) {
                    pend_st[npend] = st;
                    pend_kb[npend] = kb;
                    ++npend;
                } else if (lane == 0) {
                    tma_2d(sb, &p.tmB, kb * kBK, p.b_row0, &full[st]);
                }
                issued |= 1u << st;
                last_ph = (last_ph & ~(1u << st)) | ((uint32_t)ph << st);
                if (++st == kStages) { st = 0; ph ^= 1; }
            }
            if (!okw) break;
        }
        if (!waited) release();
        // on abort, wait (bounded) until the last fill of every stage has landed, so no copy
        // this warp issued can arrive after the CTA retires; a short sleep stays as the margin
        // for a mode-2/3 stage whose row gathers were never issued (its barrier cannot complete,
        // though the B tile has landed long before the bounded wait ends)
        if (lane == 0 && *abort_flag) {
            for (int s = 0; s < kStages; ++s) {
                if (!((issued >> s) & 1u)) continue;
                const unsigned long long t0 = now_ns();
                while (!ub_try(&full[s], (last_ph >> s) & 1u) && now_ns() - t0 < kUDrainNs) {}
            }
            const unsigned long long t0 = now_ns();
            while (now_ns() - t0 < 200000ull) {}
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------- row gathers (modes 2, 3)
        // Mode 2: 256 threads copy the stage's 128 table rows of W1 (128 bytes each) with 16-byte
        // cp.async into the same 128-byte swizzled image a TMA tile would leave (16-byte
        // chunk c of row r at r*128 + ((c ^ (r & 7)) << 4)); eight consecutive lanes cover
        // one row.  Each thread commits one group per stage and, kLag - 1 stages later, once
        // that group has landed, fences it into the async proxy and arrives on the stage's
        // full barrier.
        if (p.mode >= 2) {
            constexpr int kLag = 4;                      // stages in flight per thread (kStages >= 4)
            const int t = threadIdx.x - 6 * 32;          // 0..255
            const int c = t & 7;
            int st = 0, ph = 0, lag_st[kLag] = {0, 0, 0, 0}, nlag = 0;
            bool okg = true;
            // mode 3 (FC2): K block kb is table rows kb*64..+63 of W2T, each contributing its 128
            // output columns of this tile (two 64-column blocks 8 KB apart, K-row r of a block at
            // r*128 with the same 128-byte swizzle); 16 consecutive lanes cover one row's 256 bytes.
            // Lane t copies chunk (t & 15) of rows t/16 + 16 i.  Rows past U read row 0 (their
            // activations are zero), entries outside [0, n) too (FC1 latched them).
            const int ch = t & 15, mb = ch >> 3, c3 = ch & 7;
            auto fc2_rows = [&](int kb, const char** rows) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = kb * kBK + i * 16 + (t >> 4);
                    int j = r < q.K ? q.tab[r] : 0;
                    j = (unsigned)j < (unsigned)p.n ? j : 0;
                    rows[i] = reinterpret_cast<const char*>(p.W) + (size_t)j * p.d * 2;
                }
            };
            for (int u = blockIdx.x; u < units && okg; u += gridDim.x) {
                const int tile = u / q.splits, sp = u % q.splits;
                const int kb0 = (int)((long long)sp * q.kblocks / q.splits);
                const int kb1 = (int)((long long)(sp + 1) * q.kblocks / q.splits);
                // mode 2: rows 32 i + t / 8 of the tile; a table entry outside [0, n) is latched
                // and read as row 0 (its activation is zero)
                const char* rows[4];
                if (p.mode == 2) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = tile * kBM + i * 32 + (t >> 3);
                        int j = r < q.M ? q.tab[r] : 0;
                        if ((unsigned)j >= (unsigned)p.n) { atomicOr(p.err, ERR_IDX_RANGE); j = 0; }
                        rows[i] = reinterpret_cast<const char*>(p.W) + (size_t)j * p.d * 2 + c * 16;
                    }
                } else if (kb0 < kb1) {
                    fc2_rows(kb0, rows);
                }
                const size_t col3 = ((size_t)tile * kBM + mb * 64 + c3 * 8) * 2;   // mode 3 byte column
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!ub_wait(&empty[st], ph ^ 1, abort_flag, p.err)) { okg = false; break; }
                    char* sa = base + st * kStageBytes;
                    if (p.mode == 2) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int r = i * 32 + (t >> 3);
                            cp_async16(sa + r * 128 + ((c ^ (r & 7)) << 4), rows[i] + (size_t)kb * kBK * 2);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int r = i * 16 + (t >> 4);
                            cp_async16(sa + mb * 8192 + r * 128 + ((c3 ^ (r & 7)) << 4), rows[i] + col3);
                        }
                        if (kb + 1 < kb1) fc2_rows(kb + 1, rows);      // next block's rows, off the copy path
                    }
                    cp_async_commit();
                    lag_st[nlag++] = st;
                    if (nlag == kLag) {
                        // all but the newest kLag - 1 groups have landed: signal the oldest stage
                        cp_async_wait<kLag - 1>();
                        fence_async_smem();
                        ub_arrive(&full[lag_st[0]]);
#pragma unroll
                        for (int i = 0; i + 1 < kLag; ++i) lag_st[i] = lag_st[i + 1];
                        nlag = kLag - 1;
                    }
                    if (++st == kStages) { st = 0; ph ^= 1; }
                }
            }
            if (t == 0) UTRACE(6);
            // land and signal what is still in flight
            cp_async_wait<0>();
            fence_async_smem();
            for (int i = 0; i < nlag; ++i) ub_arrive(&full[lag_st[i]]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer (one thread)
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | ((uint32_t)p.dtype << 7) | ((uint32_t)p.dtype << 10) |
                                   ((p.mode == 3 ? 1u : 0u) << 15) | ((uint32_t)(N >> 3) << 17) |
                                   ((uint32_t)(kBM >> 4) << 24);
            int st = 0, ph = 0, ab = 0, aph = 0;
            bool issued = false;
            for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
                const int sp = u % q.splits;
                const int kb0 = (int)((long long)sp * q.kblocks / q.splits);
                const int kb1 = (int)((long long)(sp + 1) * q.kblocks / q.splits);
                if (kb1 == kb0) continue;
                if (!ub_wait(&tempty[ab], aph ^ 1, abort_flag, p.err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(ab * N);
                bool okm = true;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!ub_wait(&full[st], ph, abort_flag, p.err)) { okm = false; break; }
                    if (!issued && kb == kb0) UTRACE(2);
                    tc_fence_after();
                    const uint32_t sa = s32(base + st * kStageBytes), sb = sa + 16384u;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        const uint64_t adesc = p.mode == 3 ? sdesc(sa + k * 2048u, 512u, 64u)
                                                           : sdesc(sa + k * 32u, 1u, 64u);
                        const uint64_t bdesc = sdesc(sb + k * 32u, 1u, 64u);
                        umma(d_tmem, adesc, bdesc, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    ucommit(&empty[st]);
                    issued = true;
                    if (++st == kStages) { st = 0; ph ^= 1; }
                }
                if (!okm) break;
                ucommit(&tfull[ab]);
                if (++ab == 2) { ab = 0; aph ^= 1; }
            }
            UTRACE(3);
            // every MMA issued by this thread has completed before TMEM is released
            if (issued) {
                ucommit(done);
                const unsigned long long t0 = now_ns();
                while (!ub_try(done, 0) && now_ns() - t0 < kUWaitNs) {}
            }
        }
    } else if (warp >= 2 && warp <= 5) {
        // ------------------------------------------------------------- epilogue (warps 2..5)
        // The accumulator row is read from TMEM 16 columns at a time (with the matching
        // lo chunk in modes 1 and 3), so registers do not grow with N.
        const int quad = warp & 3;               // TMEM lanes 32*quad .. 32*quad+31
        const int lane_row = quad * 32 + lane;
        const int et = threadIdx.x - 64;         // 0..127
        volatile int no_abort = 0;
        int ab = 0, aph = 0;
        const bool pair = p.mode == 1 || p.mode == 3;
        const int half = pair ? p.Gt : N;        // columns of one half, a multiple of 16
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            const int tile = u / q.splits, sp = u % q.splits;
            const int kb0 = (int)((long long)sp * q.kblocks / q.splits);
            const int kb1 = (int)((long long)(sp + 1) * q.kblocks / q.splits);
            const bool has = kb1 > kb0;
            // loaded while the accumulators are still being computed: the row's bias and
            // state (this thread's row, or its first kPre reduction items under split-K)
            constexpr int kPre = 4;
            const int r0 = kBM * sp / q.splits, nrows = kBM * (sp + 1) / q.splits - r0;
            const int items = nrows * (half / 4);
            float pre_b[kPre];
            int pre_s[kPre];
            const bool gsplit = q.splits > 1 && p.cluster <= 1;
            const uint32_t gbase = gsplit && et == 0 ? __ldcg(&p.tickets[kTicketBase + tile]) : 0u;
            if (q.splits == 1) {
                pre_s[0] = row_pre<T>(p, q, tile, lane_row, pre_b[0]);
            } else {
#pragma unroll
                for (int k = 0; k < kPre; ++k) {
                    const int it = et + 128 * k;
                    pre_s[k] = it < items ? row_pre<T>(p, q, tile, r0 + it / (half / 4), pre_b[k]) : 0;
                }
            }
            uint32_t taddr = 0;
            if (has) {
                // time bound only: all four epilogue warps leave this wait the same way
                if (!ub_wait(&tfull[ab], aph, &no_abort, p.err)) break;
                tc_fence_after();
                taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(ab * N);
            }
            if (q.splits == 1) {
                bool any = false;
                for (int c0 = 0; c0 < half; c0 += 16) {
                    float hi[16], lo[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) hi[i] = lo[i] = 0.f;
                    if (has) {
                        tmem_ld16(taddr + c0, hi);
                        if (pair) tmem_ld16(taddr + half + c0, lo);
                        tmem_wait_ld();
                    }
                    finish_chunk<T>(p, tile, lane_row, c0, hi, lo, &any, 16, pre_s[0], pre_b[0]);
                }
                if (p.mode == 1) {                   // one mask word per 32 rows
                    const uint32_t bits = __ballot_sync(0xffffffffu, any);
                    const int word = (tile * kBM + (lane_row & ~31)) >> 5;
                    if (lane == 0 && word < (p.n >> 5)) {
                        if (p.mask_or) atomicOr(&p.mask[word], bits);
                        else p.mask[word] = bits;
                    }
                }
            } else if (p.cluster > 1) {
                // split-K in a cluster: this row goes to the reduction buffer of the CTA that owns
                // it (rows rank * rpo ..), slot [sp][row - owner's first row]
                const uint32_t owner = (uint32_t)(lane_row / p.rpo);
                const uint32_t slot = s32(base + p.red_off) +
                                      (uint32_t)(((sp * p.rpo + (lane_row - (int)owner * p.rpo)) * N) * 4);
                const uint32_t dst = cluster_map(slot, owner);
                for (int c0 = 0; c0 < N; c0 += 16) {
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.f;
                    if (has) {
                        tmem_ld16(taddr + c0, v);
                        tmem_wait_ld();
                    }
#pragma unroll
                    for (int c = 0; c < 16; c += 4) cluster_st4(dst + (uint32_t)(c0 + c) * 4u, v[c], v[c + 1], v[c + 2], v[c + 3]);
                }
            } else {
                // split-K: publish this split's partial
                float* mine = p.partial + ((size_t)u * kBM + lane_row) * N;
                for (int c0 = 0; c0 < N; c0 += 16) {
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.f;
                    if (has) {
                        tmem_ld16(taddr + c0, v);
                        tmem_wait_ld();
                    }
#pragma unroll
                    for (int c = 0; c < 16; c += 4)
                        __stcg(reinterpret_cast<float4*>(mine + c0 + c), make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]));
                }
            }
            if (has) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) ub_arrive(&tempty[ab]);
                if (++ab == 2) { ab = 0; aph ^= 1; }
                if (et == 0) UTRACE(4);
            }
            if (q.splits == 1 || p.cluster > 1) continue;
            // split-K: once every split of the tile has published its partial, the CTA of
            // split sp sums its share of the tile's rows (rows sp kBM / splits ..) over all
            // splits, in split order.  The epilogue threads' partial stores are ordered by the
            // barrier before one release add to the tile's arrival count; the count reaching
            // base + splits (an acquire, then the barrier) makes every split's partial visible.
            // All splits' CTAs are resident, one unit per CTA, so the wait is for work already
            // running; it is bounded all the same.  Split 0 then records the new base for the
            // next call, after every split has read the old one.
            epi_sync();
            if (et == 0) {
                const uint32_t target = gbase + (uint32_t)q.splits;
                red_release_add_u32(&p.tickets[kTicketArrive + tile], 1u);
                const unsigned long long t0 = now_ns();
                bool okr = true;
                while ((int32_t)(ld_acquire_u32(&p.tickets[kTicketArrive + tile]) - target) < 0) {
                    if (now_ns() - t0 > kUWaitNs) {
                        atomicOr(p.err, ERR_PIPE_TIMEOUT);
                        okr = false;
                        break;
                    }
                }
                if (sp == 0) __stcg(&p.tickets[kTicketBase + tile], target);
                *s_go = okr;
            }
            epi_sync();
            if (*s_go) {
                const size_t sstride = (size_t)kBM * N;
                auto add4 = [](float* a, const float4& w) { a[0] += w.x; a[1] += w.y; a[2] += w.z; a[3] += w.w; };
                // thread item it: row it / (half / 4) of the share, columns 4 (it % (half / 4)) ..
                auto reduce_item = [&](int it, int state, float bias) {
                    const int row = r0 + it / (half / 4), c0 = (it % (half / 4)) * 4;
                    const float* src = p.partial + ((size_t)tile * q.splits * kBM + row) * N + c0;
                    float hi[4] = {0.f, 0.f, 0.f, 0.f}, lo[4] = {0.f, 0.f, 0.f, 0.f};
                    // four splits' loads out together, summed in split order
                    for (int s0 = 0; s0 < q.splits; s0 += 4) {
                        const int ns = min(4, q.splits - s0);
                        float4 a[4], b[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float* sk = src + (size_t)(s0 + (k < ns ? k : 0)) * sstride;
                            a[k] = __ldcg(reinterpret_cast<const float4*>(sk));
                            b[k] = pair ? __ldcg(reinterpret_cast<const float4*>(sk + half)) : make_float4(0.f, 0.f, 0.f, 0.f);
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            if (k < ns) {
                                add4(hi, a[k]);
                                add4(lo, b[k]);
                            }
                        }
                    }
                    bool any = false;
                    finish_chunk<T>(p, tile, row, c0, hi, lo, &any, 4, state, bias);
                };
#pragma unroll
                for (int k = 0; k < kPre; ++k) {
                    const int it = et + 128 * k;
                    if (it < items) reduce_item(it, pre_s[k], pre_b[k]);
                }
                for (int it = et + 128 * kPre; it < items; it += 128) {
                    float bias;
                    const int state = row_pre<T>(p, q, tile, r0 + it / (half / 4), bias);
                    reduce_item(it, state, bias);
                }
            }
        }
        if (p.mode == 1 && p.cidx) {
            // the CTA whose mask words land last compacts the union mask into the ascending
            // neuron table, with all its threads, after the final barrier (no separate launch).
            // The barrier orders this CTA's mask words before one acquire-release count: the
            // last CTA to count sees every CTA's words.
            epi_sync();
            if (et == 0) *s_go = atom_acq_rel_add_u32(&p.tickets[kTicketCompact], 1u) == gridDim.x - 1;
        }
        if (et == 0) UTRACE(5);
    }
    __syncwarp();
    if (p.cluster > 1) {
        // every split of the tile has written its rows to their owners: reduce this CTA's
        // rows over the splits in split order, all threads sharing (row, 4-column) items
        cluster_sync_all();
        const int S = p.cluster, rank = blockIdx.x % S, tile = blockIdx.x / S;
        const bool pair = p.mode == 3;
        const int half = pair ? p.Gt : N;
        const int r0 = rank * p.rpo, nrows = max(0, min(kBM, r0 + p.rpo) - r0);
        const int nc4 = half / 4;
        const float* red = reinterpret_cast<const float*>(base + p.red_off);
        if (blockIdx.x < q.tiles * S) {
            for (int it = threadIdx.x; it < nrows * nc4; it += kUThreads) {
                const int rr = it / nc4, c0 = (it % nc4) * 4;
                float hi[4] = {0.f, 0.f, 0.f, 0.f}, lo[4] = {0.f, 0.f, 0.f, 0.f};
                for (int sp = 0; sp < S; ++sp) {
                    const float* src = red + ((size_t)(sp * p.rpo + rr) * N + c0);
                    const float4 a = *reinterpret_cast<const float4*>(src);
                    hi[0] += a.x; hi[1] += a.y; hi[2] += a.z; hi[3] += a.w;
                    if (pair) {
                        const float4 b = *reinterpret_cast<const float4*>(src + half);
                        lo[0] += b.x; lo[1] += b.y; lo[2] += b.z; lo[3] += b.w;
                    }
                }
                float bias;
                const int state = row_pre<T>(p, q, tile, r0 + rr, bias);
                bool any = false;
                finish_chunk<T>(p, tile, r0 + rr, c0, hi, lo, &any, 4, state, bias);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols));
    }
    if (p.mode == 1 && p.cidx && *s_go) {                 // uniform over the CTA
        compact_mask_cta(p.mask, p.n >> 5, p.cidx, p.ccount, p.ccount2, s_wsum);
        if (threadIdx.x == 0) p.tickets[kTicketCompact] = 0u;     // ready for the next call
    }
    if (threadIdx.x == 0) UTRACE(7);
}

// stage ring and TMEM allocation for an MMA of N columns
void size_launch(UParams& p) {
    p.stage_bytes = 16384 + p.N * 128;
    const int red_bytes = p.cluster > 1 ? p.cluster * p.rpo * p.N * 4 : 0;
    p.stages = std::min(kMaxStages, (200 * 1024 - red_bytes - 1024) / p.stage_bytes);
    p.red_off = p.stages * p.stage_bytes + 1024;
    int cols = 32;
    while (cols < 2 * p.N) cols *= 2;
    p.tmem_cols = cols;
}

// Trace slots: launch i since the trace buffer was bound writes slot i mod (slots held).
// Every slot is as wide as the SM count, whatever the launch's own grid, so that launches of
// different grids (clustered or not) never overlap.
unsigned g_utrace_seq = 0;
const void* g_utrace_buf = nullptr;

unsigned long long* trace_slot(int grid) {
    if (!trace_bytes()) return nullptr;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return nullptr;
    const size_t per = (size_t)std::max(grid, sms) * kUTraceMarks * sizeof(unsigned long long);
    void* buf = trace_buffer(per);
    if (!buf) return nullptr;
    if (buf != g_utrace_buf) {
        g_utrace_buf = buf;
        g_utrace_seq = 0;
    }
    const size_t slots = trace_bytes() / per;
    return static_cast<unsigned long long*>(buf) + (size_t)(g_utrace_seq++ % slots) * (per / sizeof(unsigned long long));
}

cudaError_t launch(UParams& p, int grid, cudaStream_t st) {
    size_launch(p);
    p.trace = trace_slot(grid);
    if (p.N > kMaxN || p.stages < 2) return cudaErrorInvalidValue;
    // the kernel rounds the dynamic region's start up to 1024 bytes: with a reduction buffer,
    // its end (red_off + red_bytes past that start) keeps a full 1024 bytes of slack
    const size_t red_bytes = p.cluster > 1 ? (size_t)p.cluster * p.rpo * p.N * 4 : 0;
    const size_t smem = red_bytes ? (size_t)p.red_off + red_bytes + 1024
                                  : (size_t)p.stages * p.stage_bytes + 1024 + 256;
    auto kern = p.dtype == SPFFN_BF16 ? k_umma<__nv_bfloat16> : k_umma<__half>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the kernel may start while the previous one drains
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kUThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (p.cluster > 1) {
        if (grid % p.cluster) return cudaErrorInvalidValue;
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)p.cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, kern, p);
}

// Split-K through distributed shared memory: the S = splits of each of `tiles` tiles form
// one cluster (S <= 8, the portable cluster size; N <= 64 keeps the reduction buffer small).
// Returns the grid (tiles x S), or 0 when the global-memory split reduction is used.
int use_cluster(UParams& p, int tiles, int splits) {
    const int S = std::min(splits, kMaxCluster);
    if (S < 2 || p.N > 64 || tiles * S > p.G) return 0;
    p.cluster = S;
    p.rpo = (kBM + S - 1) / S;
    return tiles * S;
}

UParams base_params(const spffn_ctx& c, int B) {
    UParams p;
    memset(&p, 0, sizeof(p));
    p.B = B;
    p.dtype = c.cfg.dtype;
    p.n = c.cfg.n; p.d = c.cfg.d; p.H = c.cfg.H;
    p.G = c.num_sms;
    p.partial = c.upartial();
    p.tickets = c.utickets();
    p.err = &c.ctl()->err;
    return p;
}

}  // namespace

// Token groups of the split-activation modes: B tokens in ceil(B / 128) groups of
// Gt tokens (a multiple of 16); group g's hi rows start at 2 g Gt, its lo rows at
// 2 g Gt + Gt, so one B-operand box of 2 Gt rows covers a group.
UnionGroups union_groups(int B) {
    UnionGroups u;
    u.groups = (B + kGroup - 1) / kGroup;
    u.Gt = round16((B + u.groups - 1) / u.groups);
    return u;
}

bool union_fused_compaction(const spffn_ctx& c) { return c.cfg.n / 32 <= kCompactWords * kUThreads; }

bool union_supported(const spffn_ctx& c, int B) {
    return B >= kUStackMinBatch && B <= kMaxBatch && B <= c.cfg.max_batch && c.cfg.d % 128 == 0 && c.lay.upartial != 0 &&
           c.num_sms <= kMaxUnionCtas && encoder() != nullptr;
}

cudaError_t union_predict(const spffn_ctx& c, const void* x, int B, int32_t* idx, int32_t* count, int32_t* count2,
                          cudaStream_t st, bool defer_table)
{
    defer_table = defer_table && union_fused_compaction(c);
    const auto& g = c.cfg;
    const UnionGroups ug = union_groups(B);
    // predictor layer 1: D[H x B] = Wp1 . X^T, split-K, -> h (fp32) and its hi/lo pairs
    UParams p = base_params(c, B);
    p.mode = 0;
    p.N = round16(B);
    p.M = g.H;
    p.K = g.d;
    p.Gs = ug.Gt;
    const int tiles = (g.H + kBM - 1) / kBM;
    const int kblocks = g.d / kBK;
    p.splits_fixed = std::max(1, std::min(kblocks, c.num_sms / tiles));
    // splits of under 8 K blocks reduce through a cluster (their hand-off outweighs their
    // streaming); longer ones keep all CTAs busy with the global reduction (measured: OPT-13B
    // shape, 18 splits of ~4 blocks, 2.55 -> 2.39 ms per step at B = 16; OPT-66B shape, 9
    // splits of 16 blocks, 6.35 -> 6.81 ms with a cluster of 8)
    const int grid0 = kblocks < 8 * p.splits_fixed ? use_cluster(p, tiles, p.splits_fixed) : 0;
    if (grid0) p.splits_fixed = p.cluster;
    p.bias = c.w.bp1;
    p.out_split = c.hsplit();
    p.out_f32 = c.h();
    if (!make_map(&p.tmA, c.w.Wp1, g.dtype, g.H, g.d, kBM)) return cudaErrorInvalidValue;
    if (!make_map(&p.tmB, x, g.dtype, B, g.d, p.N)) return cudaErrorInvalidValue;
    cudaError_t e = launch(p, grid0 ? grid0 : c.num_sms, st);
    if (e != cudaSuccess) return e;
    // predictor layer 2, one token group at a time: D[n x 2Gt] = Wp2 . hsplit_g^T -> union mask words
    for (int gi = 0; gi < ug.groups; ++gi) {
        UParams q = base_params(c, B);
        q.mode = 1;
        q.N = 2 * ug.Gt;
        q.M = g.n;
        q.K = g.H;
        q.Gt = ug.Gt;
        q.Bt = std::min(ug.Gt, B - gi * ug.Gt);
        q.b_row0 = 2 * gi * ug.Gt;
        q.mask_or = gi > 0;
        q.bias = c.w.bp2;
        q.mask = c.mask();
        if (gi == ug.groups - 1 && union_fused_compaction(c) && !defer_table) {
            q.cidx = idx;
            q.ccount = count;
            q.ccount2 = count2;
        }
        if (!make_map(&q.tmA, c.w.Wp2, g.dtype, g.n, g.H, kBM)) return cudaErrorInvalidValue;
        if (!make_map(&q.tmB, c.hsplit(), g.dtype, 2 * ug.groups * ug.Gt, g.H, q.N)) return cudaErrorInvalidValue;
        e = launch(q, c.num_sms, st);
        if (e != cudaSuccess) return e;
    }
    if (!union_fused_compaction(c)) return launch_compact(c, idx, count, count2, st);
    return cudaSuccess;
}

cudaError_t union_forward(const spffn_ctx& c, const void* x, int B, const int32_t* idx, const int32_t* count,
                          float* y, cudaStream_t st, int32_t* table_out, int32_t* count2)
{
    if (table_out && (table_out != idx || !union_fused_compaction(c))) return cudaErrorInvalidValue;
    const auto& g = c.cfg;
    const UnionGroups ug = union_groups(B);
    // FC1 over the table rows: D[U x B] = W1[table] . X^T -> a (hi/lo pairs), zeros past U
    UParams p = base_params(c, B);
    p.mode = 2;
    p.N = round16(B);
    p.K = g.d;
    p.Gs = ug.Gt;
    p.count = count;
    p.idx = idx;
    if (table_out) {
        p.mask = c.mask();
        p.tpriv = c.utab();
        p.cidx = table_out;
        p.ccount = const_cast<int32_t*>(count);
        p.ccount2 = count2;
    }
    p.bias = c.w.b1;
    p.out_split = c.asplit();
    p.W = c.w.W1;
    if (!make_map(&p.tmB, x, g.dtype, B, g.d, p.N)) return cudaErrorInvalidValue;
    cudaError_t e = launch(p, c.num_sms, st);
    if (e != cudaSuccess) return e;
    // FC2, one token group at a time: D[d x 2Gt] = W2T[table]^T . asplit_g^T -> y
    for (int gi = 0; gi < ug.groups; ++gi) {
        UParams q = base_params(c, B);
        q.mode = 3;
        q.N = 2 * ug.Gt;
        q.M = g.d;
        q.Gt = ug.Gt;
        q.Bt = std::min(ug.Gt, B - gi * ug.Gt);
        q.t_base = gi * ug.Gt;
        q.b_row0 = 2 * gi * ug.Gt;
        q.count = count;
        q.idx = idx;
        q.bias = c.w.b2;
        q.out_f32 = y;
        q.W = c.w.W2T;
        const int tiles3 = (g.d + kBM - 1) / kBM;
        const int grid3 = use_cluster(q, tiles3, c.num_sms / tiles3);
        if (!make_map(&q.tmB, c.asplit(), g.dtype, 2 * ug.groups * ug.Gt, g.n, q.N)) return cudaErrorInvalidValue;
        e = launch(q, grid3 ? grid3 : c.num_sms, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace spffn
