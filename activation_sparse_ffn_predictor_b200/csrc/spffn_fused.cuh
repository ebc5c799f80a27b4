// Persistent whole-stack decode kernel (spffn_fused.cu).
#pragma once
#include "spffn_internal.cuh"

namespace spffn {
bool fused_decode_supported(spffn_ctx* const* layers, int L, int B);
bool fused_tables_supported(spffn_ctx* const* layers, int L, int B);
// lookahead: the neuron set of layer l+1 is predicted from x_l (layer 0 from x_0)
cudaError_t launch_fused_decode(spffn_ctx* const* layers, int L, const void* x_in, int B, void* x_out, float* y,
                                int32_t* counts, bool lookahead, cudaStream_t st);
// caller-supplied neuron tables, no predictor: tabs[l] / tab_counts[l] are device pointers
cudaError_t launch_fused_tables(spffn_ctx* const* layers, int L, const void* x_in, int B,
                                const int32_t* const* tabs, const int32_t* const* tab_counts, void* x_out,
                                float* y, int32_t* counts, cudaStream_t st);
void set_trace(void* buf, size_t bytes);
int trace_marks();
}  // namespace spffn
