// Union-mask tensor-core path (spffn_union.cu).
#pragma once
#include "spffn_internal.cuh"

namespace spffn {
struct UnionGroups {
    int groups, Gt;   // token groups of the split-activation modes, tokens per group (multiple of 16)
};
UnionGroups union_groups(int B);
bool union_supported(const spffn_ctx& c, int B);
// the table is compacted inside the last logits launch (else by a launch of its own)
bool union_fused_compaction(const spffn_ctx& c);
cudaError_t union_predict(const spffn_ctx& c, const void* x, int B, int32_t* idx, int32_t* count, int32_t* count2,
                          cudaStream_t st);
cudaError_t union_forward(const spffn_ctx& c, const void* x, int B, const int32_t* idx, const int32_t* count,
                          float* y, cudaStream_t st);
cudaError_t launch_compact(const spffn_ctx& c, int32_t* idx, int32_t* count, int32_t* count2, cudaStream_t st);
// whole stack in one persistent launch on the union path (3 <= B <= 128, same shape in every layer)
bool ustack_supported(spffn_ctx* const* layers, int L, int B);
// process-wide: 0 per-layer launches, 1 the whole-stack kernel wherever it applies,
// 2 (default) the whole-stack kernel for B < 16 only
void set_ustack_mode(int mode);
int ustack_mode();
cudaError_t launch_ustack(spffn_ctx* const* layers, int L, const void* x_in, int B, void* x_out, float* y,
                          int32_t* counts, cudaStream_t st);
}  // namespace spffn
