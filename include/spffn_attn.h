/*
 * spffn_attn.h — head-sparse attention decode with an attention-head predictor
 * on one NVIDIA B200 (sm_100a), the attention half of DejaVu's contextual
 * sparsity.
 *
 * Passage that defines the operations (page title, section):
 *   [PI1] "LLM模型之PowerInfer1.0" — DejaVu appendix: equation (-1)
 *         (S_A <- SP_A(y); y~ <- MHA restricted to S_A), the head predictor
 *         (a two-layer MLP whose output layer has one unit per head, each with
 *         a sigmoid "select / do not select" decision), and the handling of
 *         KV-cache misses (a copy of every past token's input is kept; when a
 *         head that was skipped is selected, its missing K/V are computed from
 *         those stored inputs).
 *
 * One decode step of one attention layer, for one token y (storage dtype, [d]):
 *   h     = ReLU(Wa1 y + ba1)                          (fp32, [Ha])
 *   l_k   = Wa2[k] . h + ba2_k;  head k selected  <=>  l_k > 0  (sigmoid > 0.5)
 *   heads = the selected heads, ascending; count = their number
 *   Y[t]  = y                                          (t = tokens stored before)
 *   for each selected head k, every position p <= t whose K/V row is missing:
 *         K[k][p] = round(Wk_k Y[p] + bk_k),  V[k][p] = round(Wv_k Y[p] + bv_k)
 *         (Wk_k: rows k*dh .. k*dh+dh-1 of Wk; round = to the storage dtype)
 *   q_k   = Wq_k y + bq_k                              (fp32)
 *   o_k   = sum_p softmax_p(q_k . K[k][p] / sqrt(dh)) V[k][p],  p = 0..t   (fp32)
 *   out   = bo + sum over selected k of sum_i o_k[i] WoT[k*dh + i]          (fp32, [d])
 *   t     = t + 1
 * A head outside the set contributes nothing and gets no K/V row this step.
 * Every reduction has a fixed order: the same inputs give the same bits.
 *
 * Conventions are those of spffn.h: device pointers into caller-owned memory,
 * 16-byte aligned; the library allocates nothing; `stream` is a cudaStream_t
 * as void*; argument errors return before anything is enqueued; device-side
 * problems are latched in the workspace's error word.  The token position t is
 * kept on the device, so a step can be captured in a CUDA graph and replayed.
 */
#ifndef SPFFN_ATTN_H
#define SPFFN_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include "spffn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Shape of one attention layer and its head predictor.
 *   d     model width; d % 64 == 0, 64 <= d <= 16384
 *   nh    heads; 1 <= nh <= 1024
 *   dh    head width; dh % 8 == 0, 8 <= dh <= 256
 *   Ha    head-predictor hidden width; Ha % 64 == 0, 64 <= Ha <= 8192
 *   tmax  tokens the cache holds; 1 <= tmax <= 16384
 *   dtype storage type of weights, of y and of the cache
 *   flags 0 (reserved) */
typedef struct {
    int32_t d, nh, dh, Ha, tmax;
    int32_t dtype;
    uint32_t flags;
} spffn_attn_config;

/* One layer's weights: device pointers, row-major, storage dtype, borrowed until
 * spffn_attn_destroy.  Biases may be NULL (= 0).
 *   Wq, Wk, Wv [nh*dh][d]   projections; head k owns rows k*dh .. k*dh+dh-1
 *   bq, bk, bv [nh*dh]
 *   WoT        [nh*dh][d]   output projection stored head-major: row k*dh+i is
 *                           column k*dh+i of Wo, so each head is dh contiguous rows
 *   bo         [d]
 *   Wa1 [Ha][d], ba1 [Ha], Wa2 [nh][Ha], ba2 [nh]   the head predictor SP_A */
typedef struct {
    const void *Wq, *bq, *Wk, *bk, *Wv, *bv, *WoT, *bo, *Wa1, *ba1, *Wa2, *ba2;
} spffn_attn_weights;

typedef struct spffn_attn_ctx spffn_attn_ctx;

/* Device pointers into a context's cache, for inspection (read-only use):
 *   K, V    [nh][tmax][dh] storage dtype; a row exists where filled is 1
 *   filled  [nh][tmax] uint8
 *   Y       [tmax][d] storage dtype: the stored token inputs
 *   t       device int32: tokens stored so far */
typedef struct {
    const void* K;
    const void* V;
    const uint8_t* filled;
    const void* Y;
    const int32_t* t;
} spffn_attn_cache_view;

/* Bytes of device workspace (cache included) a context with this config needs,
 * 0 on a bad config.  Pure host function. */
size_t spffn_attn_workspace_bytes(const spffn_attn_config* cfg);

/* Validate, bind the caller's workspace (device, >= spffn_attn_workspace_bytes,
 * 256-byte aligned, zero-filled by the caller: an empty cache), return a new
 * host-side context.  Enqueues nothing. */
spffn_status spffn_attn_create(const spffn_attn_config* cfg, const spffn_attn_weights* w, void* workspace,
                               size_t workspace_bytes, spffn_attn_ctx** out);

/* Free the host-side context.  Safe on NULL. */
spffn_status spffn_attn_destroy(spffn_attn_ctx* ctx);

/* Empty the cache (t = 0, no K/V rows) on `stream`. */
spffn_status spffn_attn_reset(spffn_attn_ctx* ctx, void* stream);

/* One decode step (see the top of this file).  y: device [d] storage dtype.
 * heads: device int32 [nh] (the selected heads, ascending, first *count
 * entries); count: device int32 scalar; out: device fp32 [d].  When the cache
 * is full (t == tmax) the step latches SPFFN_ERR_DEVICE_CHECK, selects no
 * head, stores nothing and writes out = bo. */
spffn_status spffn_attn_step(spffn_attn_ctx* ctx, const void* y, int32_t* heads, int32_t* count, float* out,
                             void* stream);

/* The context's cache (pure host function). */
spffn_status spffn_attn_cache(spffn_attn_ctx* ctx, spffn_attn_cache_view* view);

/* Number of kernels one spffn_attn_step enqueues. */
int32_t spffn_attn_step_kernel_launches(void);

/* Read and clear the context's device error word (synchronises `stream`);
 * SPFFN_OK if clean, else SPFFN_ERR_DEVICE_CHECK; *code may be NULL. */
spffn_status spffn_attn_last_device_error(spffn_attn_ctx* ctx, uint32_t* code, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPFFN_ATTN_H */
