// Mean-pooled key pyramid (paper §Pyramid): leaves are the mean of C raw
// keys, every higher level the unweighted mean of the (one or two) children
// a block has.
//
// HBM-bound: every key is read once with 16-byte coalesced loads and summed
// in fp32; each pyramid row is written once. The leaf pass also builds the
// first kSubLevels levels above the leaves inside the CTA (from shared
// memory); upper passes then fold 2^kUpperLevels nodes per CTA until the
// root. One cooperative launch runs every pass, with grid-wide barriers
// between them, so a small pyramid costs one launch, not one per pass. All
// passes use the same two-child mean so that every route to a row (batch
// build, decode init, decode append) produces identical bits.
#include <cooperative_groups.h>

#include "pyramid.cuh"

namespace cg = cooperative_groups;

namespace pisa {

namespace {

constexpr int kLeafWarps = 8;    // leaves per CTA in the leaf pass (one per warp)
constexpr int kSubLevels = 3;    // log2(kLeafWarps): levels 2..4 built in-CTA
constexpr int kUpperNodes = 32;  // input nodes per CTA in an upper pass
constexpr int kUpperLevels = 5;  // log2(kUpperNodes)
constexpr int kThreads = kLeafWarps * 32;

// Tokens of sequence b: len[b] when given (clamped to the rows the cache
// holds), else the uniform count.
__device__ inline int64_t tokens_of(int64_t n_uniform, const int32_t* len, int b, int64_t k_rows) {
  const int64_t n = len ? static_cast<int64_t>(len[b]) : n_uniform;
  return n < k_rows ? n : k_rows;
}

// Leaf pass of one CTA: kLeafWarps leaves of head bh (one per warp), then the
// kSubLevels levels above them that lie inside this group, from shared memory.
template <typename T, int D>
__device__ void leaf_group(const T* __restrict__ k, float* pyr, const Layout& lay, int64_t n_uniform,
                           const int32_t* __restrict__ len, int H, int64_t k_rows, int C, const PageMap& pm, int bh,
                           int64_t group, float (*sm)[kUpperNodes][D]) {
  const int b = bh / H;
  const int64_t n = tokens_of(n_uniform, len, b, k_rows);
  const int64_t M1 = level_size(n, C, 1);
  const int64_t leaf0 = group * kLeafWarps;
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

// Upper pass of one CTA: kUpperNodes nodes of level la of head bh, folded into
// levels la+1 .. la+kUpperLevels. Level la was written by other CTAs before a
// grid-wide barrier, so it is read through L2 (__ldcg), not the read-only path.
template <int D>
__device__ void upper_group(float* pyr, const Layout& lay, int64_t n_uniform, const int32_t* __restrict__ len, int H,
                            int64_t k_rows, int C, int la, int bh, int64_t group, float (*sm)[kUpperNodes][D]) {
  const int b = bh / H;
  const int64_t n = tokens_of(n_uniform, len, b, k_rows);
  if (n <= 0) return;
  const int L = num_levels(n, C);
  if (la >= L) return;
  const int64_t Ma = level_size(n, C, la);
  const int64_t node0 = group * kUpperNodes;
  if (node0 >= Ma) return;
  float* pbh = pyr + static_cast<int64_t>(bh) * lay.R * D;
  for (int x = threadIdx.x; x < kUpperNodes * D; x += blockDim.x) {
    const int j = x / D, e = x % D;
    sm[0][j][e] = (node0 + j < Ma) ? __ldcg(pbh + (lay.off[la] + node0 + j) * D + e) : 0.f;
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

// The whole pyramid in one cooperative launch. Every CTA walks leaf groups
// grid-strided; after a grid-wide barrier the upper passes fold the level
// kSubLevels + 1 nodes kUpperLevels levels at a time, with a barrier between
// passes. n_max bounds every head's token count, so all CTAs take the same
// number of barriers.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) pyramid_kernel(const T* __restrict__ k, float* pyr, Layout lay,
                                                           int64_t n_max, int64_t n_uniform,
                                                           const int32_t* __restrict__ len, int H, int BH,
                                                           int64_t k_rows, int C, PageMap pm) {
  __shared__ __align__(16) float sm[2][kUpperNodes][D];
  const int64_t groups = (level_size(n_max, C, 1) + kLeafWarps - 1) / kLeafWarps;
  for (int64_t u = blockIdx.x; u < groups * BH; u += gridDim.x) {
    leaf_group<T, D>(k, pyr, lay, n_uniform, len, H, k_rows, C, pm, static_cast<int>(u / groups), u % groups, sm);
    __syncthreads();
  }
  const int L = num_levels(n_max, C);
  for (int la = 1 + kSubLevels; la < L; la += kUpperLevels) {
    cg::this_grid().sync();
    const int64_t ng = (level_size(n_max, C, la) + kUpperNodes - 1) / kUpperNodes;
    for (int64_t u = blockIdx.x; u < ng * BH; u += gridDim.x) {
      upper_group<D>(pyr, lay, n_uniform, len, H, k_rows, C, la, static_cast<int>(u / ng), u % ng, sm);
      __syncthreads();
    }
  }
}

int resident_ctas(const void* kern) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  return per_sm * sms;
}

template <typename T, int D>
cudaError_t build_impl(const void* k, float* pyr, const Layout& lay, int64_t n_max, int64_t n_uniform,
                       const int32_t* len, int BH, int H, int64_t k_rows, int C, PageMap pm, cudaStream_t st) {
  const int64_t groups = (level_size(n_max, C, 1) + kLeafWarps - 1) / kLeafWarps * BH;
  const void* kern = reinterpret_cast<const void*>(pyramid_kernel<T, D>);
  const int64_t cap = resident_ctas(kern);
  const unsigned grid = static_cast<unsigned>(groups < cap ? groups : cap);
  const T* kp = static_cast<const T*>(k);
  void* args[] = {&kp, &pyr, const_cast<Layout*>(&lay), &n_max, &n_uniform, &len, &H, &BH, &k_rows, &C, &pm};
  cudaError_t err;
  {
    TimedLaunch tl("pyramid_kernel", st);
    err = cudaLaunchCooperativeKernel(kern, dim3(grid), dim3(kThreads), args, 0, st);
  }
  count_launch();
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
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
