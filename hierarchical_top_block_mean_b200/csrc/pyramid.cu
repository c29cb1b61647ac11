// Mean-pooled key pyramid (paper §Pyramid): leaves are the mean of C raw
// keys, every higher level the unweighted mean of the (one or two) children
// a block has.
//
// HBM-bound: every key is read once with 16-byte coalesced loads and summed
// in fp32; each pyramid row is written once. The leaf pass also builds the
// first kSubLevels levels above the leaves inside the CTA (from shared
// memory); upper passes then fold 2^kUpperLevels nodes per CTA until the
// root. All passes use the same two-child mean so that every route to a row
// (batch build, decode init, decode append) produces identical bits.
#include "pyramid.cuh"

namespace pisa {

namespace {

constexpr int kLeafWarps = 8;    // leaves per CTA in the leaf pass (one per warp)
constexpr int kSubLevels = 3;    // log2(kLeafWarps): levels 2..4 built in-CTA
constexpr int kUpperNodes = 32;  // input nodes per CTA in an upper pass
constexpr int kUpperLevels = 5;  // log2(kUpperNodes)

// Tokens of sequence b: len[b] when given (clamped to the rows the cache
// holds), else the uniform count.
__device__ inline int64_t tokens_of(int64_t n_uniform, const int32_t* len, int b, int64_t k_rows) {
  const int64_t n = len ? static_cast<int64_t>(len[b]) : n_uniform;
  return n < k_rows ? n : k_rows;
}

template <typename T, int D>
__global__ void __launch_bounds__(kLeafWarps * 32) pyramid_leaf_kernel(const T* __restrict__ k, float* __restrict__ pyr,
                                                                       Layout lay, int64_t n_uniform,
                                                                       const int32_t* __restrict__ len, int H,
                                                                       int64_t k_rows, int C, PageMap pm) {
  __shared__ __align__(16) float sm[2][kLeafWarps][D];
  const int bh = blockIdx.y;
  const int b = bh / H;
  const int64_t n = tokens_of(n_uniform, len, b, k_rows);
  const int64_t M1 = level_size(n, C, 1);
  const int64_t leaf0 = static_cast<int64_t>(blockIdx.x) * kLeafWarps;
  if (n <= 0 || leaf0 >= M1) return;
  const int L = num_levels(n, C);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const T* kbh = k + static_cast<int64_t>(bh) * k_rows * D;
  float* pbh = pyr + static_cast<int64_t>(bh) * lay.R * D;

  const int64_t leaf = leaf0 + warp;
  if (leaf < M1) {
    float mean[LeafMean<T, D>::kVec];
    const int64_t hi = (leaf + 1) * C < n ? (leaf + 1) * C : n;
    if (pm.bt) {  // the leaf's keys are rows 0 .. of its page (same summation order)
      const int64_t page = pm.bt[static_cast<int64_t>(b) * pm.max_pages + leaf];
      leaf_mean_warp<T, D>(k + (page * H + bh % H) * C * D, 0, hi - leaf * C, mean);
    } else {
      leaf_mean_warp<T, D>(kbh, leaf * C, hi, mean);
    }
    LeafMean<T, D>::store(mean, &sm[0][warp][0], pbh + (lay.off[1] + leaf) * D, lane);
  }
  // Levels above the leaves that lie inside this CTA's subtree.
  int cur = 0;
  for (int l = 2; l <= 1 + kSubLevels && l <= L; ++l) {
    __syncthreads();
    const int64_t Mprev = level_size(n, C, l - 1);
    const int64_t Ml = level_size(n, C, l);
    const int nodes = kLeafWarps >> (l - 1);
    const int64_t node0 = leaf0 >> (l - 1);
    for (int x = threadIdx.x; x < nodes * D; x += blockDim.x) {
      const int j = x / D, e = x % D;
      const int64_t node = node0 + j;
      if (node >= Ml) continue;
      const int64_t c0 = 2 * node;
      const float a = sm[cur][2 * j][e];
      const float v = (c0 + 1 < Mprev) ? mean2(a, sm[cur][2 * j + 1][e]) : a;
      sm[cur ^ 1][j][e] = v;
      pbh[(lay.off[l] + node) * D + e] = v;
    }
    cur ^= 1;
  }
}

// Folds kUpperNodes nodes of level `la` per CTA into levels la+1 .. la+kUpperLevels.
template <int D>
__global__ void __launch_bounds__(256) pyramid_upper_kernel(float* __restrict__ pyr, Layout lay, int64_t n_uniform,
                                                            const int32_t* __restrict__ len, int H, int64_t k_rows,
                                                            int C, int la) {
  __shared__ __align__(16) float sm[2][kUpperNodes][D];
  const int bh = blockIdx.y;
  const int b = bh / H;
  const int64_t n = tokens_of(n_uniform, len, b, k_rows);
  if (n <= 0) return;
  const int L = num_levels(n, C);
  if (la >= L) return;
  const int64_t Ma = level_size(n, C, la);
  const int64_t node0 = static_cast<int64_t>(blockIdx.x) * kUpperNodes;
  if (node0 >= Ma) return;
  float* pbh = pyr + static_cast<int64_t>(bh) * lay.R * D;
  for (int x = threadIdx.x; x < kUpperNodes * D; x += blockDim.x) {
    const int j = x / D, e = x % D;
    sm[0][j][e] = (node0 + j < Ma) ? pbh[(lay.off[la] + node0 + j) * D + e] : 0.f;
  }
  int cur = 0;
  for (int l = la + 1; l <= la + kUpperLevels && l <= L; ++l) {
    __syncthreads();
    const int64_t Mprev = level_size(n, C, l - 1);
    const int64_t Ml = level_size(n, C, l);
    const int nodes = kUpperNodes >> (l - la);
    const int64_t nb = node0 >> (l - la);
    for (int x = threadIdx.x; x < nodes * D; x += blockDim.x) {
      const int j = x / D, e = x % D;
      const int64_t node = nb + j;
      if (node >= Ml) continue;
      const float a = sm[cur][2 * j][e];
      const float v = (2 * node + 1 < Mprev) ? mean2(a, sm[cur][2 * j + 1][e]) : a;
      sm[cur ^ 1][j][e] = v;
      pbh[(lay.off[l] + node) * D + e] = v;
    }
    cur ^= 1;
  }
}

template <typename T, int D>
cudaError_t build_impl(const void* k, float* pyr, const Layout& lay, int64_t n_max, int64_t n_uniform,
                       const int32_t* len, int BH, int H, int64_t k_rows, int C, PageMap pm, cudaStream_t st) {
  const int64_t M1 = level_size(n_max, C, 1);
  dim3 grid(static_cast<unsigned>((M1 + kLeafWarps - 1) / kLeafWarps), BH);
  pyramid_leaf_kernel<T, D><<<grid, kLeafWarps * 32, 0, st>>>(static_cast<const T*>(k), pyr, lay, n_uniform, len, H,
                                                               k_rows, C, pm);
  count_launch();
  cudaError_t err = cudaGetLastError();
  const int L = num_levels(n_max, C);
  for (int la = 1 + kSubLevels; la < L && err == cudaSuccess; la += kUpperLevels) {
    const int64_t Ma = level_size(n_max, C, la);
    dim3 g2(static_cast<unsigned>((Ma + kUpperNodes - 1) / kUpperNodes), BH);
    pyramid_upper_kernel<D><<<g2, 256, 0, st>>>(pyr, lay, n_uniform, len, H, k_rows, C, la);
    count_launch();
    err = cudaGetLastError();
  }
  return err;
}

}  // namespace

cudaError_t launch_build_pyramid(int dtype, int D, const void* k, float* pyr, const Layout& lay, int64_t n_max,
                                 int64_t n_uniform, const int32_t* len, int BH, int H, int64_t k_rows, int C,
                                 cudaStream_t st, PageMap pm) {
  if (dtype == PISA_DTYPE_BF16) {
    if (D == 128) return build_impl<bf16, 128>(k, pyr, lay, n_max, n_uniform, len, BH, H, k_rows, C, pm, st);
    return build_impl<bf16, 64>(k, pyr, lay, n_max, n_uniform, len, BH, H, k_rows, C, pm, st);
  }
  if (D == 128) return build_impl<float, 128>(k, pyr, lay, n_max, n_uniform, len, BH, H, k_rows, C, pm, st);
  return build_impl<float, 64>(k, pyr, lay, n_max, n_uniform, len, BH, H, k_rows, C, pm, st);
}

}  // namespace pisa
