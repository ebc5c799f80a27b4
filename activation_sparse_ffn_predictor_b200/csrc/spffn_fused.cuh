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
// testing aid for the bounded-wait failure path (process-wide): limit of the grid-barrier
// waits of later persistent launches (0 = the default 2 s) and an unmeetable grid barrier
void set_wait_test(unsigned long long limit_ns, bool unmeetable_barrier);
unsigned long long wait_test_ns();        // current grid-barrier wait limit of the persistent kernels
uint32_t wait_test_bar_extra();           // extra arrivals their grid barriers expect (0 or 1)
void* trace_buffer(size_t need);          // the bound trace buffer if at least `need` bytes, else null
size_t trace_bytes();                     // bytes of the bound trace buffer (0 if none)
// hot-neuron L2 residency (process-wide): rows per dealt range copied with evict_last (0 = off)
void set_l2_hot_rows(int rows);
int l2_hot_rows();
}  // namespace spffn
