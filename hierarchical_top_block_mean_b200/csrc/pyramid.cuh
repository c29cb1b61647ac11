// Pyramid building blocks shared by the batch build and the decode update.
#pragma once

#include "common.cuh"

namespace pisa {

// Mean of two children as stored at every level above the leaves. One
// definition for every writer keeps batch, init and append bit-identical.
__device__ inline float mean2(float a, float b) { return (a + b) * 0.5f; }

// Lane layout for summing key rows with 16-byte loads: each lane owns kVec
// consecutive columns of every kRpw-th row.
template <typename T, int D>
struct LeafMean {
  static constexpr int kVec = 16 / static_cast<int>(sizeof(T));
  static constexpr int kLpr = D / kVec;  // lanes per key row
  static constexpr int kRpw = 32 / kLpr; // rows per warp-wide load
  static_assert(kLpr <= 32 && 32 % kLpr == 0, "row must fit a warp");

  // Lanes [0, kLpr) hold the finished mean of columns [lane*kVec, +kVec).
  static __device__ void store(const float* mean, float* sm_row, float* g_row, int lane) {
    if (lane < kLpr) {
#pragma unroll
      for (int e = 0; e < kVec; e += 4) {
        float4 v = make_float4(mean[e], mean[e + 1], mean[e + 2], mean[e + 3]);
        if (sm_row) *reinterpret_cast<float4*>(sm_row + lane * kVec + e) = v;
        *reinterpret_cast<float4*>(g_row + lane * kVec + e) = v;
      }
    }
  }
};

// Adds 16 bytes of key elements (4 fp32 or 8 bf16), already loaded, to acc.
__device__ inline void add16(uint4 u, const float*, float* acc) {
  acc[0] += __uint_as_float(u.x);
  acc[1] += __uint_as_float(u.y);
  acc[2] += __uint_as_float(u.z);
  acc[3] += __uint_as_float(u.w);
}
__device__ inline void add16(uint4 u, const bf16*, float* acc) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
  }
}
// Plain (coherent) loads: callers may read rows that the same kernel has just
// written, or rows in shared memory.
template <typename T>
__device__ inline void add16(const T* p, float* acc) {
  add16(*reinterpret_cast<const uint4*>(p), p, acc);
}

// Mean of key rows [lo, hi) of one head (rows of D elements), computed by one
// warp in fp32: each lane sums its rows in order, then the row groups are
// combined by a fixed butterfly, then divided by the row count.
template <typename T, int D>
__device__ inline void leaf_mean_warp(const T* __restrict__ kbh, int64_t lo, int64_t hi,
                                      float* mean /*[LeafMean<T,D>::kVec]*/) {
  using LM = LeafMean<T, D>;
  const int lane = threadIdx.x & 31;
  const int col = (lane % LM::kLpr) * LM::kVec;
  float acc[LM::kVec];
#pragma unroll
  for (int e = 0; e < LM::kVec; ++e) acc[e] = 0.f;
  int64_t j = lo + lane / LM::kLpr;
  // Batches of kBatch loads in flight, then their adds in row order (the
  // summation order is that of a plain row-by-row loop).
  constexpr int kBatch = 8;
  for (; j + (kBatch - 1) * LM::kRpw < hi; j += kBatch * LM::kRpw) {
    uint4 u[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) u[i] = *reinterpret_cast<const uint4*>(kbh + (j + i * LM::kRpw) * D + col);
#pragma unroll
    for (int i = 0; i < kBatch; ++i) add16(u[i], kbh, acc);
  }
  for (; j < hi; j += LM::kRpw) add16(kbh + j * D + col, acc);
#pragma unroll
  for (int o = LM::kLpr; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < LM::kVec; ++e) acc[e] += __shfl_xor_sync(kFull, acc[e], o);
  const float cnt = static_cast<float>(hi - lo);
#pragma unroll
  for (int e = 0; e < LM::kVec; ++e) mean[e] = acc[e] / cnt;
}

// Key rows held in pages: page bt[b * max_pages + i] holds the C keys of leaf
// i of sequence b for every head, as [H][C][D] rows. bt == nullptr: dense
// [B, H, k_rows, D] keys.
struct PageMap {
  const int32_t* bt;
  int max_pages;
};

// Builds pyr for every (b, h) over its first n_b tokens (n_b = len[b] when len
// is given, else n_uniform) into a layout sized for lay; k has k_rows rows per
// head. n_max bounds every n_b.
cudaError_t launch_build_pyramid(int dtype, int D, const void* k, float* pyr, const Layout& lay, int64_t n_max,
                                 int64_t n_uniform, const int32_t* len, int BH, int H, int64_t k_rows, int C,
                                 cudaStream_t st, PageMap pm = PageMap{nullptr, 0});

}  // namespace pisa
