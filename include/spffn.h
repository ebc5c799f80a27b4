/*
 * spffn.h — activation-sparse FFN decoding on one NVIDIA B200 (sm_100a).
 *
 * A ReLU FFN block  y = W2 ReLU(W1 x + b1) + b2  is decoded activation-sparsely:
 * a two-layer X-H-O MLP predictor scores every FFN neuron, the neurons whose
 * sigmoid output exceeds 0.5 (logit > 0) are compacted into an ascending
 * neuron table, and only those rows of W1 and of the neuron-major W2T = W2^T
 * are read and computed.
 *
 * Passages that define the operations (page title, section):
 *   [PI1] "LLM模型之PowerInfer1.0" — §2.1 (FFN: FC1, ReLU gate, FC2), §3.2
 *         (single-layer example, Figure 3), §4.1 (adaptive sparse predictor,
 *         X-H-O MLP), §4.2 (neuron tables), §4.4 (neuron-aware operators),
 *         §5.1 (offline profiler counting activations), §5.2 equation (1)
 *         (impact = activation frequency), DejaVu appendix equation (-1)
 *         (predict S_M, then MLP restricted to S_M), closing question 3 (AXPY
 *         over contiguous neuron columns for the down projection).
 *   [SPX] "Técnicas dispersas para una aceleración 100X en la inferencia de
 *         modelos de lenguaje grandes" — batch size erodes the sparsity
 *         (union of per-token sets), 128-byte memory blocks.
 *
 * Conventions (all entry points):
 *   - Every pointer argument named as "device" is a device pointer into memory
 *     owned by the caller (e.g. allocated with the PyTorch caching allocator)
 *     and must be 16-byte aligned.  The library never allocates device memory:
 *     scratch lives in a caller-provided workspace.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every device call is asynchronous on `stream`; none syncs the
 *     host, none copies device->host.
 *   - Argument errors are detected on the host and returned before anything is
 *     enqueued.  CUDA launch errors return SPFFN_ERR_CUDA.  Data-dependent
 *     problems found on the device (e.g. a caller-supplied count > n) are
 *     clamped, latched in the workspace's error word, and reported by
 *     spffn_last_device_error.  No device code traps or spins without bound.
 *   - One context is used by one stream at a time.  Contexts that share a
 *     workspace must not run concurrently.
 *   - No C++ exception crosses this interface.
 */
#ifndef SPFFN_H
#define SPFFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPFFN_OK = 0,
    SPFFN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or shape */
    SPFFN_ERR_UNSUPPORTED = 2,   /* valid request this build does not serve (no sm_100 device) */
    SPFFN_ERR_WORKSPACE = 3,     /* workspace missing or smaller than spffn_workspace_bytes() */
    SPFFN_ERR_CUDA = 4,          /* a CUDA runtime call failed */
    SPFFN_ERR_DEVICE_CHECK = 5,  /* a device-side check latched an error (see spffn_last_device_error) */
    SPFFN_ERR_TIMEOUT = 6        /* a bounded device wait gave up */
} spffn_status;

typedef enum { SPFFN_F16 = 0, SPFFN_BF16 = 1 } spffn_dtype;

/* Shape of one FFN layer and its predictor.
 *   d          model width; d % 64 == 0, 64 <= d <= 16384
 *   n          FFN neurons;  n % 32 == 0, 32 <= n <= 131072
 *   H          predictor hidden width; H % 64 == 0, 64 <= H <= 8192
 *   max_batch  largest batch B the context will see; 1 <= max_batch <= 256.  Batches
 *              of 16..256 tokens run on the union tensor-core path, which needs
 *              d % 128 == 0; without it a batch above 32 is SPFFN_ERR_UNSUPPORTED
 *   dtype      storage type of weights and of x (accumulation is always fp32)
 *   flags      0 (reserved) */
typedef struct {
    int32_t d, n, H, max_batch;
    int32_t dtype;
    uint32_t flags;
} spffn_config;

/* One layer's weights: device pointers, row-major, storage dtype, borrowed
 * until spffn_destroy.
 *   W1  [n][d]   FC1 rows (row j = neuron j)
 *   b1  [n]      FC1 bias
 *   W2T [n][d]   FC2 stored neuron-major: row j = column j of W2 ([PI1]
 *                closing question 3), so each neuron is one contiguous row
 *   b2  [d]      FC2 bias, may be NULL (= 0)
 *   Wp1 [H][d]   predictor layer 1;  bp1 [H] may be NULL (= 0)
 *   Wp2 [n][H]   predictor layer 2;  bp2 [n] may be NULL (= 0) */
typedef struct {
    const void *W1, *b1, *W2T, *b2, *Wp1, *bp1, *Wp2, *bp2;
} spffn_weights;

typedef struct spffn_ctx spffn_ctx;

/* Bytes of device workspace a context with this config needs (0 on a bad
 * config).  Pure host function. */
size_t spffn_workspace_bytes(const spffn_config* cfg);

/* Validate `cfg` and `w`, bind the caller's workspace (device, >=
 * spffn_workspace_bytes(cfg) bytes, 256-byte aligned, zero-filled by the
 * caller before first use, borrowed until spffn_destroy), and return a new
 * host-side context in *out.  Enqueues nothing.  Kernels initialise every
 * scratch word they read except the latched error word, which starts from the
 * caller's zero fill and is cleared by spffn_last_device_error. */
spffn_status spffn_create(const spffn_config* cfg, const spffn_weights* w, void* workspace,
                          size_t workspace_bytes, spffn_ctx** out);

/* Free the host-side context.  Safe on NULL.  Does not touch device memory. */
spffn_status spffn_destroy(spffn_ctx* ctx);

/* Predictor + threshold + compaction ([PI1] §4.1, DejaVu appendix (-1);
 * [PI1] §4.2 neuron table; batch union per [SPX]):
 *   h_t   = ReLU(Wp1 x_t + bp1)                  (fp32)
 *   l_t,i = Wp2[i] . h_t + bp2_i                 (fp32)
 *   neuron i selected  <=>  l_t,i > 0 for some token t  (sigmoid > 0.5)
 *   idx[0..count) = selected neurons, ascending; *count written on device.
 * x: device [B][d] storage dtype; 1 <= B <= max_batch (B > 32 only on the union
 * path, see spffn_config; else SPFFN_ERR_UNSUPPORTED).
 * idx: device int32, capacity n.  count: device int32 scalar. */
spffn_status spffn_predict(spffn_ctx* ctx, const void* x, int32_t B,
                           int32_t* idx, int32_t* count, void* stream);

/* Neuron-aware FFN over a neuron table ([PI1] §4.4 vec_dot for FC1, AXPY
 * over neuron-major rows for FC2):
 *   y_t = b2 + sum over j in idx[0..count), ascending, of ReLU(W1[j].x_t + b1_j) W2T[j]
 * computed as fixed per-chunk fp32 partial sums reduced in a fixed order
 * (deterministic: same inputs give the same bits).  Every token is computed
 * on every neuron of the table.
 * idx/count: device, e.g. from spffn_predict or any caller mask; entries must
 * be in [0,n) (out-of-range entries are skipped and latched as a device
 * error) and *count is clamped to n (latched).  count == 0 gives y = b2.
 * y: device fp32 [B][d]. */
spffn_status spffn_forward(spffn_ctx* ctx, const void* x, int32_t B, const int32_t* idx,
                           const int32_t* count, float* y, void* stream);

/* spffn_predict followed by spffn_forward on the same x (one layer's decode). */
spffn_status spffn_step(spffn_ctx* ctx, const void* x, int32_t B, int32_t* idx, int32_t* count,
                        float* y, void* stream);

/* Layer chaining used between stacked layers (the pages give no attention or
 * norm; this is the library's stated choice):
 *   x_next_t = round_dtype( (x_t + y_t) / sqrt(mean_c (x_t + y_t)_c^2 + 1e-6) )
 * x, x_next: device [B][d] storage dtype (may not alias); y: device fp32 [B][d]. */
spffn_status spffn_chain(spffn_ctx* ctx, const void* x, const float* y, int32_t B, void* x_next,
                         void* stream);

/* One decode step through a stack of L layers: for l = 0..L-1
 *   (idx_l, count_l) = predict_l(x_l);  y_l = forward_l(x_l);  x_{l+1} = chain(x_l, y_l)
 * layers: host array of L contexts with equal d, dtype and max_batch.
 * x_in: device [B][d]; x_out: device [B][d] = x_L; y: device fp32 [B][d] = y_{L-1};
 * counts: device int32 [L] (count_l), may be NULL.  Intermediate x_l live in
 * the layers' workspaces. */
spffn_status spffn_decode(spffn_ctx* const* layers, int32_t L, const void* x_in, int32_t B,
                          void* x_out, float* y, int32_t* counts, void* stream);

/* spffn_decode with look-ahead prediction (DejaVu's asynchronous predictor,
 * equation (-2) in the DejaVu appendix of "LLM模型之PowerInfer1.0"): the
 * neuron set of layer l+1 is predicted from layer l's input, so the predictor
 * of the next layer runs beside the FFN of this one:
 *   (idx_0, count_0) = predict_0(x_0)
 *   for l = 0..L-1:  (idx_{l+1}, count_{l+1}) = predict_{l+1}(x_l)   [l+1 < L]
 *                    y_l = forward_l(x_l; idx_l);  x_{l+1} = chain(x_l, y_l)
 * Layer l+1's own predictor weights (Wp1, bp1, Wp2, bp2 of layers[l+1]) are the
 * ones applied to x_l.  Arguments, outputs and errors as for spffn_decode. */
spffn_status spffn_decode_lookahead(spffn_ctx* const* layers, int32_t L, const void* x_in, int32_t B,
                                    void* x_out, float* y, int32_t* counts, void* stream);

/* One decode step through L layers on caller-supplied neuron tables, no predictor
 * (e.g. each token's true activation set, or any other mask):
 *   for l = 0..L-1:  y_l = forward_l(x_l; tables[l][0..tab_counts[l]));  x_{l+1} = chain(x_l, y_l)
 * tables: host array of L device pointers to int32 tables, entries as for
 * spffn_forward (distinct, in [0,n); out-of-range entries skipped and latched).
 * tab_counts: device int32 [L] (each clamped to [0,n], latched).  x_in, x_out,
 * y, counts (which receives the clamped lengths, may be NULL) as for
 * spffn_decode.  At B <= 2 the whole stack is one persistent kernel (two grid
 * barriers per layer); otherwise per-layer launches. */
spffn_status spffn_decode_tables(spffn_ctx* const* layers, int32_t L, const void* x_in, int32_t B,
                                 const int32_t* const* tables, const int32_t* tab_counts, void* x_out, float* y,
                                 int32_t* counts, void* stream);

/* Device pointer to the neuron table that the last spffn_decode or
 * spffn_decode_lookahead left in this layer's workspace (ascending neuron
 * indices; its length is that call's counts[l]).  Valid until the next call
 * that uses ctx.  Pure host function; INVALID_ARG on a NULL argument. */
spffn_status spffn_layer_table(spffn_ctx* ctx, const int32_t** idx);

/* Number of kernels one spffn_decode (or spffn_decode_lookahead) call with these
 * arguments enqueues (the persistent whole-stack kernel: 1; otherwise per layer
 * 4 + 2 x the union path's token groups, ceil(B / 128), or 6 off that path), 0 on
 * bad arguments.
 * Pure host function. */
int32_t spffn_decode_kernel_launches(spffn_ctx* const* layers, int32_t L, int32_t B);

/* Offline profiler ([PI1] §5.1): for T profiling tokens X [T][d] (device,
 * storage dtype), counts[j] += #{t : W1[j].X_t + b1_j > 0}.  counts: device
 * uint32 [n], accumulated (caller zeroes it before the first batch). */
spffn_status spffn_profile_counts(spffn_ctx* ctx, const void* X, int32_t T, uint32_t* counts,
                                  void* stream);

/* Hot-first placement ([PI1] §5.2 equation (1), impact = frequency): host
 * arrays; perm[s] = original neuron placed in slot s, ordering by count
 * descending, ties by original index ascending.  Pure host function. */
spffn_status spffn_reorder(const uint32_t* counts_host, int32_t n, int32_t* perm_host);

/* Hot-first placement dealt over `parts` contiguous slot ranges (range c =
 * slots [floor(n c / parts), floor(n (c+1) / parts))): neurons in hot-first
 * order (as spffn_reorder) are dealt round-robin, the i-th hottest going to
 * range i mod parts, filling each range in ascending slots.  With parts =
 * spffn_num_partials(), every CTA of the whole-stack decode kernel owns a range
 * with the same expected activity.  Pure host function. */
spffn_status spffn_reorder_dealt(const uint32_t* counts_host, int32_t n, int32_t parts, int32_t* perm_host);

/* Row gather applying a neuron table: dst row s = src row perm[s], for `rows`
 * rows of `row_bytes` bytes (row_bytes % 16 == 0).  src, dst, perm: device;
 * dst must not alias src; perm entries must lie in [0, rows) (out-of-range
 * rows are left unwritten).  Permutes W1, W2T and Wp2 into hot-first order;
 * 2-byte bias vectors use spffn_permute_vector. */
spffn_status spffn_permute_rows(const void* src, void* dst, int32_t rows, int32_t row_bytes,
                                const int32_t* perm, void* stream);

/* Element gather dst[s] = src[perm[s]] for a vector of 2-byte elements. */
spffn_status spffn_permute_vector(const void* src, void* dst, int32_t count, const int32_t* perm,
                                  void* stream);

/* Tracing aid: bind a device buffer (or NULL to unbind) into which later
 * whole-stack decode launches write %globaltimer stamps (u64 nanoseconds),
 * laid out [CTA][layer][spffn_trace_marks()], at fixed points of each layer:
 * 0 input formed, 1 first predictor-1 chunk ready, 2 hidden layer done,
 * 3 after barrier, 4 h loaded, 5 first predictor-2 chunk ready, 6 own
 * neuron list final, 7 first FFN rows ready, 8 FFN partial written, 9 after
 * barrier, 10 reduction and table written, 11 after barrier, 12 fourth
 * predictor-2 chunk ready, 13 fourth chunk's rows computed by every warp, 14 last
 * predictor-2 chunk ready, 15 last chunk's rows computed (thread 0).
 * A mark a CTA does not reach in a layer (no rows or no neurons) stays 0.
 * The union path's per-layer tensor-core launches (batches of 16 or more) write
 * [launch slot][CTA][8] instead, slot i for the i-th such launch since the buffer
 * was bound (modulo the slots it holds): 0 set up, 1 past the wait for the
 * previous kernel, 2 first stage consumed, 3 last MMA issued, 4 last accumulator
 * read, 5 epilogue done, 6 row gathers issued, 7 exit.  A CUDA graph keeps the
 * slots of the launches it captured.
 * Buffers smaller than that are ignored.  Process-wide; not thread-safe. */
spffn_status spffn_set_trace(void* buf, size_t bytes);
int32_t spffn_trace_marks(void);

/* Selects how spffn_decode runs 3 <= B <= 128 (B <= max_batch, d % 128 == 0,
 * every layer of one shape, at most 64 layers, no look-ahead):
 *   1  the whole stack as one persistent launch on the union tensor-core path,
 *      with the weights of the next phase streaming across its grid barriers;
 *   0  per-layer launches (the tensor-core kernels of spffn_predict and
 *      spffn_forward plus the chaining for every layer, chained by programmatic
 *      dependent launch; the per-phase kernels where the union path does not
 *      apply);
 *   2  (the default) the faster of the two on the measured shapes, which is 0
 *      at every batch from 3 to 128.
 * Both compute the same function; their fp32 reductions run in different
 * orders, so results agree to rounding.  Process-wide; applies to calls made
 * afterwards; INVALID_ARG outside 0..2.  spffn_union_stack returns the mode. */
spffn_status spffn_set_union_stack(int32_t mode);
int32_t spffn_union_stack(void);

/* Hot-neuron L2 residency ([PI1] §5.2 equation (1): a neuron's impact is its
 * activation frequency; §5.3 places the most impactful neurons in the faster
 * memory).  On one GPU the faster tier is the L2 cache.  After the hot-first
 * placement dealt over the SM count of ranges (spffn_reorder_dealt with parts =
 * spffn_num_partials), slot k of every range holds the (k G + c)-th hottest
 * neuron, so the first `rows_per_range` slots of all ranges are the
 * rows_per_range x G hottest neurons of the layer.  With rows_per_range > 0 the
 * persistent decode kernel at B <= 2 (spffn_decode, spffn_decode_lookahead,
 * spffn_decode_tables and spffn_forward there) copies those neurons' W1 and W2T
 * rows with an L2 evict_last policy and every other weight byte (predictor and
 * cold rows) with evict_first, per instruction: no device-wide L2 setting is
 * changed.  The hot rows of all layers should fit in L2 together:
 * rows_per_range x G x L x 4d bytes (about 77 MB for 32 layers at d = 4096 and
 * one row per range).  0 (the default) issues no hints.  Results are the same
 * bits either way.  Process-wide; applies to launches enqueued afterwards;
 * INVALID_ARG for a negative value. */
spffn_status spffn_set_l2_hot_rows(int32_t rows_per_range);
int32_t spffn_l2_hot_rows(void);

/* Testing aid for the failure path of the persistent whole-stack kernels (the
 * single launch of spffn_decode, spffn_decode_lookahead and spffn_decode_tables
 * at B <= 2, and of spffn_decode at 16 <= B <= 128 on the union path).  Every
 * wait in those kernels is bounded; on expiry the kernel latches
 * SPFFN_ERR_TIMEOUT in the error word, raises a grid-wide abort, stops issuing
 * copies, waits (bounded) for the copies it already issued and returns,
 * leaving the context usable.  This call sets, for launches enqueued after it:
 *   limit_ns            limit of each grid-barrier wait in nanoseconds (0
 *                       restores the default of 2 s; the other waits keep 2 s);
 *   unmeetable_barrier  nonzero: each grid barrier expects one arrival more
 *                       than there are CTAs, so the first one cannot complete
 *                       and its wait runs out after limit_ns.
 * A test sets a short limit and an unmeetable barrier, runs one decode, checks
 * that spffn_last_device_error reports SPFFN_ERR_TIMEOUT, then calls
 * spffn_set_wait_test(0, 0) and checks that the next decode is clean.
 * Process-wide; not thread-safe. */
spffn_status spffn_set_wait_test(uint64_t limit_ns, int32_t unmeetable_barrier);

/* Allocation-free variant of spffn_forward (the pages have no counterpart).
 * It is for callers that cannot allocate device memory, and so cannot provide
 * the workspace an spffn_ctx needs: code that runs inside another allocator's
 * arena (a cudaMalloc of its own would bypass that allocator's accounting), or
 * code under a fixed device-memory budget that is already spent on its own
 * buffers.  The caller passes only inputs and outputs; the
 * fp32 partial sums live in a fixed 1 MiB __device__ array that every GPU
 * loading this library reserves until the process exits.
 * It computes the same function as spffn_forward for the layer described by
 * `cfg`/`w` (cfg->H and cfg->max_batch are not used), always with the
 * per-phase split kernels: a fixed split of the table into partial sums, then
 * a fixed-order reduction.  spffn_forward runs other kernels at some batches
 * (the persistent kernel at B <= 2, the tensor-core union path at B >= 16), so
 * the two agree to fp32 rounding at every B, not bitwise.
 *   Limit: 1 <= B <= 32 and B * cfg->d * 4 bytes <= 1 MiB (B = 32 needs
 *   d <= 8192), else SPFFN_ERR_INVALID_ARG / SPFFN_ERR_UNSUPPORTED, checked on
 *   the host before anything is enqueued; the number of partial sums is the
 *   largest count (<= the SM count) that fits.
 *   Set-up: the first call on a device looks up the array's device address
 *   with that device current; make that first call before any stream capture.
 *   Every call shares the array and the array keeps the last call's contents
 *   (each call overwrites what it reads): calls that overlap on the GPU
 *   (different streams, or different host threads without ordering) race and
 *   must not be issued; calls on one stream are ordered and safe.
 *   Device-side checks still clamp the count and skip out-of-range entries,
 *   but this entry point does not report them.
 *   Calls no cudaMalloc, cudaFree or allocating library routine. */
spffn_status spffn_forward_noalloc(const spffn_config* cfg, const spffn_weights* w, const void* x, int32_t B,
                                   const int32_t* idx, const int32_t* count, float* y, void* stream);

/* Read and clear the context's device error word (synchronises `stream`).
 * Returns SPFFN_OK if clean, SPFFN_ERR_DEVICE_CHECK or SPFFN_ERR_TIMEOUT;
 * *code (may be NULL) receives the raw word. */
spffn_status spffn_last_device_error(spffn_ctx* ctx, uint32_t* code, void* stream);

/* Description of the CUDA error behind the calling thread's most recent
 * SPFFN_ERR_CUDA (static string). */
const char* spffn_last_cuda_error_string(void);

/* Static description of a status code. */
const char* spffn_status_string(spffn_status s);

/* Number of fp32 partial sums the forward reduction uses (its fixed split). */
int32_t spffn_num_partials(const spffn_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* SPFFN_H */
