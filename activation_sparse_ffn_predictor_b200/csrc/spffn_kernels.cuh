// Launchers for the per-phase kernels (spffn_kernels.cu).
#pragma once
#include "spffn_internal.cuh"

namespace spffn {
// defer_table / table_out: on the union path, the table of a predict-then-forward pair is
// derived inside the forward's FC1 launch (union_predict / union_forward); elsewhere ignored
// (table_out must then be idx, and the predict writes the table as usual)
cudaError_t launch_predict(const spffn_ctx& c, const void* x, int B, int32_t* idx, int32_t* count,
                           int32_t* count2, cudaStream_t st, bool defer_table = false);
cudaError_t launch_forward(const spffn_ctx& c, const void* x, int B, const int32_t* idx, const int32_t* count,
                           float* y, cudaStream_t st, int32_t* table_out = nullptr, int32_t* count2 = nullptr);
cudaError_t launch_chain(const spffn_ctx& c, const void* x, const float* y, int B, void* xn, cudaStream_t st);
cudaError_t launch_profile(const spffn_ctx& c, const void* X, int T, uint32_t* counts, cudaStream_t st);
cudaError_t launch_permute_rows(const void* src, void* dst, int rows, int row_bytes, const int32_t* perm,
                                cudaStream_t st);
cudaError_t launch_permute_vec(const void* src, void* dst, int count, const int32_t* perm, cudaStream_t st);
int ffn_token_group(const spffn_ctx& c);
// h[t][r] = ReLU(W[r] . x_t + b[r]) for an H x d weight (the predictor hidden layer; b may be null)
cudaError_t launch_hidden(int dtype, const void* W, const void* b, const void* x, int B, int d, int H, float* h,
                          int num_sms, cudaStream_t st);
cudaError_t launch_forward_scratch(const spffn_config& g, const spffn_weights& w, const void* x, int B,
                                   const int32_t* idx, const int32_t* count, float* y, float* partial, int S,
                                   uint32_t* err, cudaStream_t st);
}  // namespace spffn
