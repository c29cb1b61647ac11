// Decode path (paper §Kernels, decoding): the mean pyramid is cached; each
// new token updates only its leaf mean and the ancestors of that leaf, and
// selection runs root-to-leaf in one kernel, scoring raw key blocks at the
// leaf level.
#include "dispatch.cuh"
#include "kernels.cuh"
#include "pyramid.cuh"
#include "rowops.cuh"

namespace pisa {

namespace {

constexpr int kRowWarps = 4;

// One CTA per sequence, one warp per kv head. Writes the new k/v rows,
// recomputes the leaf that holds them over its present keys (same routine
// and order as the batch build) and walks up the ancestors, each the mean of
// its existing children. All heads read len[s] before it is incremented.
template <typename T, int D>
__global__ void decode_append_kernel(DecodeArgs a, Layout lay, const T* __restrict__ k_new,
                                     const T* __restrict__ v_new, T* __restrict__ kc, T* __restrict__ vc,
                                     float* __restrict__ pyr, int32_t* __restrict__ len, int32_t* status) {
  using LM = LeafMean<T, D>;
  __shared__ int64_t off[kMaxLevels + 2];
  load_offsets(lay, off);
  const int s = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int64_t n = len[s];
  __syncthreads();
  if (n >= a.cap || n < 0) {
    if (threadIdx.x == 0) *status = PISA_ERR_CAPACITY;
    return;
  }
  const int64_t leaf = n / a.C;
  const int L = num_levels(n + 1, a.C);
  for (int h = warp; h < a.H_kv; h += nw) {
    const int64_t bh = static_cast<int64_t>(s) * a.H_kv + h;
    T* krow = kc + (bh * a.cap + n) * D;
    T* vrow = vc + (bh * a.cap + n) * D;
    for (int e = lane; e < D; e += 32) {
      krow[e] = k_new[bh * D + e];
      vrow[e] = v_new[bh * D + e];
    }
    __threadfence_block();
    __syncwarp();
    float mean[LM::kVec];
    leaf_mean_warp<T, D>(kc + bh * a.cap * D, leaf * a.C, n + 1, mean);
    float* P = pyr + bh * lay.R * D;
    LM::store(mean, nullptr, P + (off[1] + leaf) * D, lane);
    int64_t node = leaf;
    for (int l = 2; l <= L; ++l) {
      const int64_t sib = node ^ 1;
      const bool has_sib = sib < level_size(n + 1, a.C, l - 1);
      if (lane < LM::kLpr && has_sib) {
        const float* srow = P + (off[l - 1] + sib) * D + lane * LM::kVec;
#pragma unroll
        for (int e = 0; e < LM::kVec; ++e) mean[e] = mean2(mean[e], srow[e]);
      }
      node >>= 1;
      LM::store(mean, nullptr, P + (off[l] + node) * D, lane);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) len[s] = static_cast<int32_t>(n + 1);
}

// One warp per (sequence, kv head): selection for the query at position
// len[s] - 1 (every block of the sequence is valid for it) and/or attention.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kRowWarps * 32)
    decode_rows_kernel(DecodeArgs a, Layout lay, int mode, const T* __restrict__ q_new, const T* __restrict__ kc,
                       const T* __restrict__ vc, const float* __restrict__ pyr, const int32_t* __restrict__ len,
                       int32_t* __restrict__ sel, T* __restrict__ out, float* __restrict__ lse) {
  constexpr int kCols = D / 32;
  __shared__ __align__(16) float qs[kRowWarps][G][D];
  __shared__ int tmp[kRowWarps][32];
  __shared__ float ps[kRowWarps][G * 32];
  __shared__ int blk[kRowWarps][kMaxK];
  __shared__ int64_t off[kMaxLevels + 2];
  load_offsets(lay, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowWarps + warp;
  if (row >= static_cast<int64_t>(a.S) * a.H_kv) return;
  const int64_t s = row / a.H_kv, h = row % a.H_kv;
  const int64_t n = len[s];
  if (n <= 0 || n > a.cap) return;
  const int64_t t = n - 1;
  stage_q<T, D, G>(q_new + (s * a.H_q + h * G) * D, D, &qs[warp][0][0]);
  const T* krows = kc + row * a.cap * D;
  if (mode & 1) {
    SelectRow<T, D, G> sr{&qs[warp][0][0], pyr + row * lay.R * D, off, krows, n, t, a.C, a.K, true, a.scale,
                          tmp[warp]};
    int leaf;
    float sc;
    sr.run(leaf, sc);
    if (lane < a.K) {
      blk[warp][lane] = leaf;
      if (sel) sel[row * a.K + lane] = leaf;
    }
  } else if (lane < a.K) {
    blk[warp][lane] = sel[row * a.K + lane];
  }
  __syncwarp();
  if (mode & 2) {
    AttendRow<T, D, G> ar{&qs[warp][0][0], krows, vc + row * a.cap * D, n, t, a.C, true, a.scale, ps[warp]};
    float o[G][kCols], m[G], l[G];
    ar.run(blk[warp], a.K, o, m, l);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float inv = l[g] > 0.f ? 1.f / l[g] : 0.f;
#pragma unroll
      for (int e = 0; e < kCols; ++e) store_out(out + (s * a.H_q + h * G + g) * D + lane * kCols + e, o[g][e] * inv);
      if (lse && lane == 0) lse[s * a.H_q + h * G + g] = m[g] + logf(l[g]);
    }
  }
}

}  // namespace

cudaError_t launch_decode_append(const DecodeArgs& a, const Layout& lay, const void* k_new, const void* v_new,
                                 void* k_cache, void* v_cache, float* pyr, int32_t* len, int32_t* status,
                                 cudaStream_t st) {
  return dispatch_td(a.dtype, a.d, [&](auto tt, auto dd) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int D = decltype(dd)::value;
    const int threads = 32 * (a.H_kv < 8 ? a.H_kv : 8);
    TimedLaunch tl("decode_append_kernel", st);
    decode_append_kernel<T, D><<<a.S, threads, 0, st>>>(a, lay, static_cast<const T*>(k_new),
                                                         static_cast<const T*>(v_new), static_cast<T*>(k_cache),
                                                         static_cast<T*>(v_cache), pyr, len, status);
    count_launch();
    return cudaGetLastError();
  });
}

cudaError_t launch_decode_rows(const DecodeArgs& a, const Layout& lay, int mode, const void* q_new,
                               const void* k_cache, const void* v_cache, const float* pyr, const int32_t* len,
                               int32_t* sel, void* out, float* lse, cudaStream_t st) {
  return dispatch_tdg(a.dtype, a.d, a.H_q / a.H_kv, [&](auto tt, auto dd, auto gg) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    const unsigned blocks = static_cast<unsigned>((static_cast<int64_t>(a.S) * a.H_kv + kRowWarps - 1) / kRowWarps);
    TimedLaunch tl("decode_rows_kernel", st);
    decode_rows_kernel<T, D, G><<<blocks, kRowWarps * 32, 0, st>>>(
        a, lay, mode, static_cast<const T*>(q_new), static_cast<const T*>(k_cache), static_cast<const T*>(v_cache),
        pyr, len, sel, static_cast<T*>(out), lse);
    count_launch();
    return cudaGetLastError();
  });
}

}  // namespace pisa
