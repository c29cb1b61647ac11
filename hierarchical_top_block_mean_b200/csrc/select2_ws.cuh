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
  int32_t* rank;        // [rows][32] each candidate's position in its bucket (its count's old value)
  int32_t* bucket_off;  // [buckets + 1] exclusive scan of count
  int32_t* item_off;    // [buckets + 1] exclusive scan of ceil(count / kPairsPerItem)
  uint32_t* pairs;      // [rows * 32] (query row << 5 | slot), grouped by bucket
  uint4* planes;        // [B*H_kv][R][D/4] pyramid rows as bf16 hi/lo: {hi x4, lo x4} per 4 elements
  bf16* hi;             // [B*H_kv][R][D] bf16 hi part of each pyramid row (tensor-memory router levels), or null
  bf16* lo;             // [B*H_kv][R][D] its lo part, or null
  float* dense;         // [rows][kDenseSlots] node scores of each row's top scored levels, or null
  int32_t* item_bucket; // [items] bucket of each stage-2 work item
  int4* item_info;      // [items] {b * H_kv + h, first pair, end pair, leaf} of each work item
  int win_shift;        // query rows are bucketed by window (row >> win_shift)
  int nwin;             // windows per (b, kv head)
};

// Top scored levels by tcgen05 (G_Q = 8, d = 128, K <= 16): for each block of
// kDenseQ queries of one kv head, every node of the levels Ltop, Ltop - 1 and
// Ltop - 2 is scored at once, Ltop being the first scored level of the
// block's last query. The router reads those scores instead of gathering the
// children. Slots per row: Ltop's nodes from 0 (at most 2K <= 32), Ltop - 1's
// from 32 (at most 64), Ltop - 2's from 96 (at most 128).
constexpr int kDenseQ = 16;
constexpr int kDenseSlots = 224;
__host__ __device__ inline int dense_slot0(int i) { return i == 0 ? 0 : (i == 1 ? 32 : 96); }
// First scored level of the search for a query at position t: the highest
// level with more than K usable blocks (0 when the leaf level has <= K).
__device__ inline int start_level(int64_t n, int C, int K, int64_t t, bool causal) {
  int l = num_levels(n, C);
  while (l >= 1 && valid_count(n, C, l, t, causal) <= K) --l;
  return l;
}
bool router_top_supported(const PrefillArgs& a);
cudaError_t launch_router_top(const PrefillArgs& a, const void* q, const Layout& lay, const Ws& ws, cudaStream_t st);

// Stage-2 leaf scorer on tcgen05 tensor cores (G_Q = 8, d = 128, C = 64).
bool leaf_umma_supported(const PrefillArgs& a);
cudaError_t launch_leaf_umma(const PrefillArgs& a, const void* q, const void* k, const Ws& ws, int nb, int M1,
                             cudaStream_t st);

}  // namespace pisa
