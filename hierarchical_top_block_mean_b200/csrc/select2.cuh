// Two-stage prefill selection for bf16 (paper §Kernels): stage 1 routes levels
// L..2 per (kv head, query); stage 2 groups (query, candidate leaf) pairs by
// leaf, scores each leaf's raw keys against tiles of queries on tensor cores,
// and a final pass keeps the top K per row.
#pragma once

#include "kernels.cuh"

namespace pisa {

size_t select2_workspace_bytes(const PrefillArgs& a);
cudaError_t launch_select2(const PrefillArgs& a, const void* q, const void* k, const float* pyr, const Layout& lay,
                           int32_t* sel, float* sel_score, void* ws, cudaStream_t st);

}  // namespace pisa
