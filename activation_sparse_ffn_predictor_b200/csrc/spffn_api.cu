// C-ABI of the sparse-FFN decode library (declarations and contracts in include/spffn.h).
#include <algorithm>
#include <new>
#include <numeric>
#include <vector>
#include "spffn_internal.cuh"
#include "spffn_kernels.cuh"
#include "spffn_fused.cuh"
#include "spffn_union.cuh"

using namespace spffn;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Batches above the per-phase kernels' limit run only on the union tensor-core path.
bool batch_supported(const spffn_ctx& c, int B) { return B <= kMaxPhaseBatch || union_supported(c, B); }

bool valid_config(const spffn_config* c) {
    if (!c) return false;
    if (c->d < 64 || c->d > 16384 || c->d % 64) return false;
    if (c->n < 32 || c->n > 131072 || c->n % 32) return false;
    if (c->H < 64 || c->H > 8192 || c->H % 64) return false;
    if (c->max_batch < 1 || c->max_batch > kMaxBatch) return false;
    if (c->dtype != SPFFN_F16 && c->dtype != SPFFN_BF16) return false;
    if (c->flags != 0) return false;
    return true;
}

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        cudaGetLastError();
        return 148;
    }
    return sms;
}

thread_local cudaError_t t_last_cuda = cudaSuccess;

spffn_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return SPFFN_OK;
    t_last_cuda = e;
    return SPFFN_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* spffn_last_cuda_error_string(void) {
    return t_last_cuda == cudaSuccess ? "no CUDA error recorded" : cudaGetErrorString(t_last_cuda);
}

const char* spffn_status_string(spffn_status s) {
    switch (s) {
        case SPFFN_OK: return "ok";
        case SPFFN_ERR_INVALID_ARG: return "invalid argument";
        case SPFFN_ERR_UNSUPPORTED: return "unsupported";
        case SPFFN_ERR_WORKSPACE: return "workspace missing or too small";
        case SPFFN_ERR_CUDA: return "CUDA runtime error";
        case SPFFN_ERR_DEVICE_CHECK: return "device-side check failed";
        case SPFFN_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

size_t spffn_workspace_bytes(const spffn_config* cfg) {
    if (!valid_config(cfg)) return 0;
    return make_layout(*cfg, device_sms()).total;
}

spffn_status spffn_create(const spffn_config* cfg, const spffn_weights* w, void* workspace,
                          size_t workspace_bytes, spffn_ctx** out) {
    if (!out) return SPFFN_ERR_INVALID_ARG;
    *out = nullptr;
    if (!valid_config(cfg) || !w) return SPFFN_ERR_INVALID_ARG;
    if (!w->W1 || !w->b1 || !w->W2T || !w->Wp1 || !w->Wp2) return SPFFN_ERR_INVALID_ARG;
    const void* all[] = {w->W1, w->b1, w->W2T, w->b2, w->Wp1, w->bp1, w->Wp2, w->bp2};
    for (const void* p : all)
        if (p && !aligned16(p)) return SPFFN_ERR_INVALID_ARG;
    const int sms = device_sms();
    Layout lay = make_layout(*cfg, sms);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SPFFN_ERR_WORKSPACE;
    if (workspace_bytes < lay.total) return SPFFN_ERR_WORKSPACE;
    spffn_ctx* c = new (std::nothrow) spffn_ctx();
    if (!c) return SPFFN_ERR_UNSUPPORTED;
    c->cfg = *cfg;
    c->w = *w;
    c->ws = static_cast<char*>(workspace);
    c->ws_bytes = workspace_bytes;
    c->lay = lay;
    c->num_sms = sms;
    c->device = 0;
    cudaGetDevice(&c->device);
    cudaGetLastError();
    *out = c;
    return SPFFN_OK;
}

spffn_status spffn_destroy(spffn_ctx* ctx) {
    delete ctx;
    return SPFFN_OK;
}

int32_t spffn_num_partials(const spffn_ctx* ctx) { return ctx ? ctx->lay.S : 0; }

spffn_status spffn_predict(spffn_ctx* ctx, const void* x, int32_t B, int32_t* idx, int32_t* count,
                           void* stream) {
    if (!ctx || !x || !idx || !count || B < 1 || B > ctx->cfg.max_batch) return SPFFN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(idx)) return SPFFN_ERR_INVALID_ARG;
    if (!batch_supported(*ctx, B)) return SPFFN_ERR_UNSUPPORTED;
    return cuda_status(launch_predict(*ctx, x, B, idx, count, nullptr, (cudaStream_t)stream));
}

spffn_status spffn_forward(spffn_ctx* ctx, const void* x, int32_t B, const int32_t* idx,
                           const int32_t* count, float* y, void* stream) {
    if (!ctx || !x || !idx || !count || !y || B < 1 || B > ctx->cfg.max_batch) return SPFFN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return SPFFN_ERR_INVALID_ARG;
    if (!batch_supported(*ctx, B)) return SPFFN_ERR_UNSUPPORTED;
    spffn_ctx* one[1] = {ctx};
    if (fused_tables_supported(one, 1, B)) {
        // one persistent launch: gathered rows, FC1 + AXPY, fixed-order reduction
        const int32_t* tabs[1] = {idx};
        const int32_t* cnts[1] = {count};
        return cuda_status(launch_fused_tables(one, 1, x, B, tabs, cnts, nullptr, y, nullptr, (cudaStream_t)stream));
    }
    return cuda_status(launch_forward(*ctx, x, B, idx, count, y, (cudaStream_t)stream));
}

spffn_status spffn_step(spffn_ctx* ctx, const void* x, int32_t B, int32_t* idx, int32_t* count, float* y,
                        void* stream) {
    spffn_status s = spffn_predict(ctx, x, B, idx, count, stream);
    if (s != SPFFN_OK) return s;
    return spffn_forward(ctx, x, B, idx, count, y, stream);
}

spffn_status spffn_chain(spffn_ctx* ctx, const void* x, const float* y, int32_t B, void* x_next,
                         void* stream) {
    if (!ctx || !x || !y || !x_next || B < 1 || B > ctx->cfg.max_batch || x == x_next)
        return SPFFN_ERR_INVALID_ARG;
    return cuda_status(launch_chain(*ctx, x, y, B, x_next, (cudaStream_t)stream));
}

namespace {

spffn_status decode_impl(spffn_ctx* const* layers, int32_t L, const void* x_in, int32_t B, void* x_out, float* y,
                         int32_t* counts, bool lookahead, void* stream) {
    if (!layers || L < 1 || !x_in || !x_out || !y) return SPFFN_ERR_INVALID_ARG;
    const spffn_ctx* l0 = layers[0];
    if (!l0) return SPFFN_ERR_INVALID_ARG;
    for (int l = 0; l < L; ++l) {
        const spffn_ctx* c = layers[l];
        if (!c || c->cfg.d != l0->cfg.d || c->cfg.dtype != l0->cfg.dtype) return SPFFN_ERR_INVALID_ARG;
        if (B < 1 || B > c->cfg.max_batch) return SPFFN_ERR_INVALID_ARG;
        if (!batch_supported(*c, B)) return SPFFN_ERR_UNSUPPORTED;
    }
    if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(y) || x_in == x_out) return SPFFN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (fused_decode_supported(layers, L, B))
        return cuda_status(launch_fused_decode(layers, L, x_in, B, x_out, y, counts, lookahead, st));
    if (!lookahead && ustack_supported(layers, L, B))
        return cuda_status(launch_ustack(layers, L, x_in, B, x_out, y, counts, st));
    const void* xcur = x_in;
    cudaError_t e = cudaSuccess;
    if (lookahead) {
        const spffn_ctx& c = *layers[0];
        e = launch_predict(c, x_in, B, c.idx(), c.count(), counts, st);
        if (e != cudaSuccess) return cuda_status(e);
    }
    for (int l = 0; l < L; ++l) {
        const spffn_ctx& c = *layers[l];
        // union path: FC1 derives the table from the mask words (no compaction tail in the
        // logits launch)
        const bool tin = !lookahead && union_supported(c, B) && union_fused_compaction(c);
        if (!lookahead) {
            e = launch_predict(c, xcur, B, c.idx(), c.count(), counts ? counts + l : nullptr, st, tin);
        } else if (l + 1 < L) {
            // the next layer's set from this layer's input
            const spffn_ctx& cn = *layers[l + 1];
            e = launch_predict(cn, xcur, B, cn.idx(), cn.count(), counts ? counts + l + 1 : nullptr, st);
        }
        if (e != cudaSuccess) return cuda_status(e);
        float* yl = (l == L - 1) ? y : c.ybuf();
        e = launch_forward(c, xcur, B, c.idx(), c.count(), yl, st, tin ? c.idx() : nullptr,
                           tin && counts ? counts + l : nullptr);
        if (e != cudaSuccess) return cuda_status(e);
        void* xn = (l == L - 1) ? x_out : c.xbuf(l & 1);
        e = launch_chain(c, xcur, yl, B, xn, st);
        if (e != cudaSuccess) return cuda_status(e);
        xcur = xn;
    }
    return SPFFN_OK;
}

}  // namespace

spffn_status spffn_decode(spffn_ctx* const* layers, int32_t L, const void* x_in, int32_t B, void* x_out,
                          float* y, int32_t* counts, void* stream) {
    return decode_impl(layers, L, x_in, B, x_out, y, counts, false, stream);
}

spffn_status spffn_decode_lookahead(spffn_ctx* const* layers, int32_t L, const void* x_in, int32_t B,
                                    void* x_out, float* y, int32_t* counts, void* stream) {
    return decode_impl(layers, L, x_in, B, x_out, y, counts, true, stream);
}

spffn_status spffn_decode_tables(spffn_ctx* const* layers, int32_t L, const void* x_in, int32_t B,
                                 const int32_t* const* tables, const int32_t* tab_counts, void* x_out, float* y,
                                 int32_t* counts, void* stream) {
    if (!layers || L < 1 || !x_in || !x_out || !y || !tables || !tab_counts) return SPFFN_ERR_INVALID_ARG;
    const spffn_ctx* l0 = layers[0];
    if (!l0) return SPFFN_ERR_INVALID_ARG;
    for (int l = 0; l < L; ++l) {
        const spffn_ctx* c = layers[l];
        if (!c || !tables[l] || c->cfg.d != l0->cfg.d || c->cfg.dtype != l0->cfg.dtype) return SPFFN_ERR_INVALID_ARG;
        if (B < 1 || B > c->cfg.max_batch) return SPFFN_ERR_INVALID_ARG;
        if (!batch_supported(*c, B)) return SPFFN_ERR_UNSUPPORTED;
    }
    if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(y) || x_in == x_out) return SPFFN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    std::vector<const int32_t*> cnt(L);
    for (int l = 0; l < L; ++l) cnt[l] = tab_counts + l;
    if (fused_tables_supported(layers, L, B))
        return cuda_status(launch_fused_tables(layers, L, x_in, B, tables, cnt.data(), x_out, y, counts, st));
    const void* xcur = x_in;
    for (int l = 0; l < L; ++l) {
        const spffn_ctx& c = *layers[l];
        float* yl = (l == L - 1) ? y : c.ybuf();
        cudaError_t e = launch_forward(c, xcur, B, tables[l], cnt[l], yl, st);
        if (e != cudaSuccess) return cuda_status(e);
        if (counts) {
            e = cudaMemcpyAsync(counts + l, cnt[l], sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
            if (e != cudaSuccess) return cuda_status(e);
        }
        void* xn = (l == L - 1) ? x_out : c.xbuf(l & 1);
        e = launch_chain(c, xcur, yl, B, xn, st);
        if (e != cudaSuccess) return cuda_status(e);
        xcur = xn;
    }
    return SPFFN_OK;
}

spffn_status spffn_layer_table(spffn_ctx* ctx, const int32_t** idx) {
    if (!ctx || !idx) return SPFFN_ERR_INVALID_ARG;
    *idx = ctx->idx();
    return SPFFN_OK;
}

int32_t spffn_decode_kernel_launches(spffn_ctx* const* layers, int32_t L, int32_t B) {
    if (!layers || L < 1 || !layers[0] || B < 1 || B > layers[0]->cfg.max_batch) return 0;
    for (int l = 0; l < L; ++l)
        if (!layers[l]) return 0;
    if (fused_decode_supported(layers, L, B) || ustack_supported(layers, L, B)) return 1;
    // per layer: predictor hidden, logits, compaction, FC1 (two launches), chaining; on the
    // union path the compaction runs inside the last logits launch and logits and FC2 run
    // once per token group
    int n = 0;
    for (int l = 0; l < L; ++l)
        n += union_supported(*layers[l], B) ? 3 + 2 * union_groups(B).groups + (union_fused_compaction(*layers[l]) ? 0 : 1)
                                            : 6;
    return n;
}

spffn_status spffn_set_trace(void* buf, size_t bytes) {
    set_trace(buf, bytes);
    return SPFFN_OK;
}

int32_t spffn_trace_marks(void) { return trace_marks(); }

spffn_status spffn_set_union_stack(int32_t mode) {
    if (mode < 0 || mode > 2) return SPFFN_ERR_INVALID_ARG;
    set_ustack_mode(mode);
    return SPFFN_OK;
}

int32_t spffn_union_stack(void) { return ustack_mode(); }

spffn_status spffn_set_l2_hot_rows(int32_t rows_per_range) {
    if (rows_per_range < 0) return SPFFN_ERR_INVALID_ARG;
    set_l2_hot_rows(rows_per_range);
    return SPFFN_OK;
}

int32_t spffn_l2_hot_rows(void) { return l2_hot_rows(); }

spffn_status spffn_set_wait_test(uint64_t limit_ns, int32_t unmeetable_barrier) {
    set_wait_test((unsigned long long)limit_ns, unmeetable_barrier != 0);
    return SPFFN_OK;
}

spffn_status spffn_profile_counts(spffn_ctx* ctx, const void* X, int32_t T, uint32_t* counts, void* stream) {
    if (!ctx || !X || !counts || T < 1 || !aligned16(X)) return SPFFN_ERR_INVALID_ARG;
    return cuda_status(launch_profile(*ctx, X, T, counts, (cudaStream_t)stream));
}

spffn_status spffn_reorder(const uint32_t* counts_host, int32_t n, int32_t* perm_host) {
    if (!counts_host || !perm_host || n < 1) return SPFFN_ERR_INVALID_ARG;
    std::vector<int32_t> p(n);
    std::iota(p.begin(), p.end(), 0);
    std::stable_sort(p.begin(), p.end(),
                     [&](int32_t a, int32_t b) { return counts_host[a] > counts_host[b]; });
    std::copy(p.begin(), p.end(), perm_host);
    return SPFFN_OK;
}

spffn_status spffn_reorder_dealt(const uint32_t* counts_host, int32_t n, int32_t parts, int32_t* perm_host) {
    if (!counts_host || !perm_host || n < 1 || parts < 1) return SPFFN_ERR_INVALID_ARG;
    std::vector<int32_t> hot(n);
    std::iota(hot.begin(), hot.end(), 0);
    std::stable_sort(hot.begin(), hot.end(),
                     [&](int32_t a, int32_t b) { return counts_host[a] > counts_host[b]; });
    std::vector<int64_t> lo(parts + 1);
    int64_t widest = 0;
    for (int c = 0; c <= parts; ++c) lo[c] = (int64_t)n * c / parts;
    for (int c = 0; c < parts; ++c) widest = std::max(widest, lo[c + 1] - lo[c]);
    int64_t next = 0;
    for (int64_t r = 0; r < widest; ++r)
        for (int c = 0; c < parts; ++c)
            if (lo[c] + r < lo[c + 1]) perm_host[lo[c] + r] = hot[next++];
    return SPFFN_OK;
}

spffn_status spffn_permute_rows(const void* src, void* dst, int32_t rows, int32_t row_bytes, const int32_t* perm,
                                void* stream) {
    if (!src || !dst || !perm || rows < 1 || row_bytes < 16 || row_bytes % 16 || src == dst)
        return SPFFN_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(dst)) return SPFFN_ERR_INVALID_ARG;
    return cuda_status(launch_permute_rows(src, dst, rows, row_bytes, perm, (cudaStream_t)stream));
}

spffn_status spffn_permute_vector(const void* src, void* dst, int32_t count, const int32_t* perm, void* stream) {
    if (!src || !dst || !perm || count < 1 || src == dst) return SPFFN_ERR_INVALID_ARG;
    return cuda_status(launch_permute_vec(src, dst, count, perm, (cudaStream_t)stream));
}

spffn_status spffn_last_device_error(spffn_ctx* ctx, uint32_t* code, void* stream) {
    if (!ctx) return SPFFN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, &ctx->ctl()->err, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return SPFFN_ERR_CUDA;
    if (cudaMemsetAsync(&ctx->ctl()->err, 0, sizeof(uint32_t), st) != cudaSuccess) return SPFFN_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SPFFN_ERR_CUDA;
    if (code) *code = v;
    if (v & (ERR_BARRIER_TIMEOUT | ERR_PIPE_TIMEOUT)) return SPFFN_ERR_TIMEOUT;
    return v ? SPFFN_ERR_DEVICE_CHECK : SPFFN_OK;
}

}  // extern "C"
