// Union-mask tensor-core path (spffn_union.cu).
#pragma once
#include "spffn_internal.cuh"

namespace spffn {
struct UnionGroups {
    int groups, Gt;   // token groups of the split-activation modes, tokens per group (multiple of 16)
};
UnionGroups union_groups(int B);
bool union_supported(const spffn_ctx& c, int B);
// the table is compacted inside the last logits launch (else by a launch of its own); the
// same bound lets the FC1 launch derive it from the mask words instead
bool union_fused_compaction(const spffn_ctx& c);
// defer_table: leave the union mask in the workspace without compacting it; the FC1 launch
// of union_forward with table_out set derives the table from it
cudaError_t union_predict(const spffn_ctx& c, const void* x, int B, int32_t* idx, int32_t* count, int32_t* count2,
                          cudaStream_t st, bool defer_table = false);
// table_out (with count2, which may be null): FC1 ranks the mask words left by a deferring
// union_predict itself and writes the table to table_out and its length to count (and count2)
cudaError_t union_forward(const spffn_ctx& c, const void* x, int B, const int32_t* idx, const int32_t* count,
                          float* y, cudaStream_t st, int32_t* table_out = nullptr, int32_t* count2 = nullptr);
cudaError_t launch_compact(const spffn_ctx& c, int32_t* idx, int32_t* count, int32_t* count2, cudaStream_t st);
// whole stack in one persistent launch on the union path (3 <= B <= 128, same shape in every layer)
bool ustack_supported(spffn_ctx* const* layers, int L, int B);
// process-wide: 0 and 2 (default) per-layer launches, 1 the whole-stack kernel wherever it applies
void set_ustack_mode(int mode);
int ustack_mode();
cudaError_t launch_ustack(spffn_ctx* const* layers, int L, const void* x_in, int B, void* x_out, float* y,
                          int32_t* counts, cudaStream_t st);
}  // namespace spffn
