// Workspace of the two-stage bf16 selection, shared by its kernels.
#pragma once

#include "kernels.cuh"

namespace pisa {

// Workspace sections (all 256-byte aligned).
struct Ws {
  int32_t* cand;        // [rows][32] candidate leaves per row after stage 1 (-1 padded)
  int32_t* ncand;       // [rows] candidates per row; -1 when stage 1 already wrote sel
  float* score;         // [rows][32] leaf score of each candidate slot
  int32_t* count;       // [buckets] pairs per (b, kv head, leaf)
  int32_t* fill;        // [buckets] scatter cursors
  int32_t* bucket_off;  // [buckets + 1] exclusive scan of count
  int32_t* item_off;    // [buckets + 1] exclusive scan of ceil(count / kPairsPerItem)
  uint32_t* pairs;      // [rows * 32] (query row << 5 | slot), grouped by bucket
  uint4* planes;        // [B*H_kv][R][D/4] pyramid rows as bf16 hi/lo: {hi x4, lo x4} per 4 elements
  int32_t* item_bucket; // [items] bucket of each stage-2 work item
  int4* item_info;      // [items] {b * H_kv + h, first pair, end pair, leaf} of each work item
  int win_shift;        // query rows are bucketed by window (row >> win_shift)
  int nwin;             // windows per (b, kv head)
};

// Stage-2 leaf scorer on tcgen05 tensor cores (G_Q = 8, d = 128, C = 64).
bool leaf_umma_supported(const PrefillArgs& a);
cudaError_t launch_leaf_umma(const PrefillArgs& a, const void* q, const void* k, const Ws& ws, int nb, int M1,
                             cudaStream_t st);

}  // namespace pisa
