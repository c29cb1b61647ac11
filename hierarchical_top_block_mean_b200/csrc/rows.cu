// Warp-per-row kernels: fused root-to-leaf selection, attention and flat
// selection over prefill rows. These are the fp32 path (FFMA in fp32, no
// TF32); bf16 prefill uses the tensor-core kernels.
#include "dispatch.cuh"
#include "kernels.cuh"
#include "rowops.cuh"

namespace pisa {

namespace {

constexpr int kRowWarps = 4;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kRowWarps * 32)
    select_rows_kernel(const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ pyr, Layout lay,
                       PrefillArgs a, int32_t* __restrict__ sel, float* __restrict__ sel_score) {
  __shared__ __align__(16) float qs[kRowWarps][G][D];
  __shared__ int tmp[kRowWarps][32];
  __shared__ int64_t off[kMaxLevels + 2];
  load_offsets(lay, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowWarps + warp;
  if (row >= static_cast<int64_t>(a.B) * a.H_kv * a.Nq) return;
  const int64_t bh = row / a.Nq, i = row % a.Nq, t = a.q0 + i;  // query row and its position
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  stage_q<T, D, G>(q + ((b * a.H_q + h * G) * a.Nq + i) * D, static_cast<int64_t>(a.Nq) * D, &qs[warp][0][0]);
  SelectRow<T, D, G> sr{&qs[warp][0][0], pyr + bh * lay.R * D, off, k + bh * a.N * D, a.N, t, a.C, a.K,
                        a.causal != 0, a.scale, tmp[warp]};
  int leaf;
  float sc;
  sr.run(leaf, sc);
  if (lane < a.K) {
    sel[row * a.K + lane] = leaf;
    if (sel_score) sel_score[row * a.K + lane] = leaf >= 0 ? sc : __int_as_float(0x7fffffff);
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kRowWarps * 32)
    attn_rows_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const int32_t* __restrict__ sel, PrefillArgs a, T* __restrict__ out, float* __restrict__ lse) {
  constexpr int kCols = D / 32;
  __shared__ __align__(16) float qs[kRowWarps][G][D];
  __shared__ float ps[kRowWarps][G * 32];
  __shared__ int blk[kRowWarps][kMaxK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowWarps + warp;
  if (row >= static_cast<int64_t>(a.B) * a.H_kv * a.Nq) return;
  const int64_t bh = row / a.Nq, i = row % a.Nq, t = a.q0 + i;  // query row and its position
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  const int64_t hs = static_cast<int64_t>(a.Nq) * D;
  const int64_t qo = ((b * a.H_q + h * G) * a.Nq + i) * D;  // head 0 of the group
  stage_q<T, D, G>(q + qo, hs, &qs[warp][0][0]);
  if (lane < a.K) blk[warp][lane] = sel[row * a.K + lane];
  __syncwarp();
  AttendRow<T, D, G> ar{&qs[warp][0][0], k + bh * a.N * D, v + bh * a.N * D, a.N, t, a.C, a.causal != 0, a.scale,
                        ps[warp]};
  float o[G][kCols], m[G], l[G];
  ar.run(blk[warp], a.K, o, m, l);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float inv = l[g] > 0.f ? 1.f / l[g] : 0.f;
#pragma unroll
    for (int e = 0; e < kCols; ++e) store_out(out + qo + g * hs + lane * kCols + e, o[g][e] * inv);
    if (lse && lane == 0) lse[(b * a.H_q + h * G + g) * a.Nq + i] = m[g] + logf(l[g]);
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kRowWarps * 32)
    flat_rows_kernel(const T* __restrict__ q, const float* __restrict__ pyr, int64_t R, PrefillArgs a,
                     int32_t* __restrict__ sel) {
  __shared__ __align__(16) float qs[kRowWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowWarps + warp;
  if (row >= static_cast<int64_t>(a.B) * a.H_kv * a.Nq) return;
  const int64_t bh = row / a.Nq, i = row % a.Nq, t = a.q0 + i;  // query row and its position
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  const int64_t hs = static_cast<int64_t>(a.Nq) * D;
  const T* qg = q + ((b * a.H_q + h * G) * a.Nq + i) * D;
  // The flat score is linear in q, so the group's heads are summed first.
  for (int e = lane * 4; e < D; e += 128) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 x = load4(qg + g * hs + e);
      s.x += x.x;
      s.y += x.y;
      s.z += x.z;
      s.w += x.w;
    }
    *reinterpret_cast<float4*>(&qs[warp][e]) = s;
  }
  __syncwarp();
  const float* leaves = pyr + bh * R * D;  // level 1 occupies rows [0, M_1)
  const int64_t nv = valid_count(a.N, a.C, 1, t, a.causal != 0);
  int idx;
  if (nv <= a.K) {
    idx = lane < nv ? lane : INT_MAX;
  } else {
    float bs = -INFINITY;
    int bi = INT_MAX;
    for (int64_t i0 = 0; i0 < nv; i0 += 32) {
      const int64_t i = i0 + lane;
      float s = -INFINITY;
      if (i < nv) {
        const float* r = leaves + i * D;
        float acc = 0.f;
#pragma unroll 8
        for (int e = 0; e < D; e += 4) acc += dot4(*reinterpret_cast<const float4*>(&qs[warp][e]), load4(r + e));
        s = a.scale * acc;
      }
      const int ii = i < nv ? static_cast<int>(i) : INT_MAX;
      const float ts = __shfl_sync(kFull, bs, a.K - 1);
      const int ti = __shfl_sync(kFull, bi, a.K - 1);
      if (__ballot_sync(kFull, ranks_before(s, ii, ts, ti)) == 0) continue;
      warp_merge_best(bs, bi, s, ii);
    }
    idx = lane < a.K ? bi : INT_MAX;
  }
  warp_sort_asc(idx);
  if (lane < a.K) sel[row * a.K + lane] = idx == INT_MAX ? -1 : idx;
}

// Exact-score flat selection for one row: every usable leaf is scored by its
// raw-key LSE summed over the group (the pyramid search's leaf score), 32
// leaves per round (one per lane), merged into the running best list.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kRowWarps * 32)
    exact_rows_kernel(const T* __restrict__ q, const T* __restrict__ k, PrefillArgs a, int32_t* __restrict__ sel) {
  __shared__ __align__(16) float qs[kRowWarps][G][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowWarps + warp;
  if (row >= static_cast<int64_t>(a.B) * a.H_kv * a.Nq) return;
  const int64_t bh = row / a.Nq, i = row % a.Nq, t = a.q0 + i;  // query row and its position
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  stage_q<T, D, G>(q + ((b * a.H_q + h * G) * a.Nq + i) * D, static_cast<int64_t>(a.Nq) * D, &qs[warp][0][0]);
  SelectRow<T, D, G> sr{&qs[warp][0][0], nullptr, nullptr, k + bh * a.N * D, a.N, t, a.C, a.K,
                        a.causal != 0, a.scale, nullptr};
  const int64_t nv = valid_count(a.N, a.C, 1, t, a.causal != 0);
  int idx;
  if (nv <= a.K) {
    idx = lane < nv ? lane : INT_MAX;
  } else {
    float bs = -INFINITY;
    int bi = INT_MAX;
    for (int64_t i0 = 0; i0 < nv; i0 += 32) {
      float s = -INFINITY;
      for (int x = 0; x < 32 && i0 + x < nv; ++x) {
        const float u = sr.leaf_score(i0 + x);
        if (lane == x) s = u;
      }
      warp_merge_best(bs, bi, s, i0 + lane < nv ? static_cast<int>(i0 + lane) : INT_MAX);
    }
    idx = lane < a.K ? bi : INT_MAX;
  }
  warp_sort_asc(idx);
  if (lane < a.K) sel[row * a.K + lane] = idx == INT_MAX ? -1 : idx;
}

inline unsigned row_blocks(const PrefillArgs& a) {
  return static_cast<unsigned>((static_cast<int64_t>(a.B) * a.H_kv * a.Nq + kRowWarps - 1) / kRowWarps);
}

}  // namespace

cudaError_t launch_select_rows(const PrefillArgs& a, const void* q, const void* k, const float* pyr,
                               const Layout& lay, int32_t* sel, float* sel_score, cudaStream_t st) {
  return dispatch_tdg(a.dtype, a.d, a.H_q / a.H_kv, [&](auto tt, auto dd, auto gg) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    TimedLaunch tl("select_rows_kernel", st);
    select_rows_kernel<T, D, G><<<row_blocks(a), kRowWarps * 32, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), pyr, lay, a, sel, sel_score);
    count_launch();
    return cudaGetLastError();
  });
}

cudaError_t launch_attn_rows(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                             void* out, float* lse, cudaStream_t st) {
  return dispatch_tdg(a.dtype, a.d, a.H_q / a.H_kv, [&](auto tt, auto dd, auto gg) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    TimedLaunch tl("attn_rows_kernel", st);
    attn_rows_kernel<T, D, G><<<row_blocks(a), kRowWarps * 32, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), sel, a, static_cast<T*>(out),
        lse);
    count_launch();
    return cudaGetLastError();
  });
}

cudaError_t launch_flat_rows(const PrefillArgs& a, const void* q, const float* pyr, int64_t R, int32_t* sel,
                             cudaStream_t st) {
  return dispatch_tdg(a.dtype, a.d, a.H_q / a.H_kv, [&](auto tt, auto dd, auto gg) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    TimedLaunch tl("flat_rows_kernel", st);
    flat_rows_kernel<T, D, G><<<row_blocks(a), kRowWarps * 32, 0, st>>>(static_cast<const T*>(q), pyr, R, a, sel);
    count_launch();
    return cudaGetLastError();
  });
}

cudaError_t launch_exact_rows(const PrefillArgs& a, const void* q, const void* k, int32_t* sel, cudaStream_t st) {
  return dispatch_tdg(a.dtype, a.d, a.H_q / a.H_kv, [&](auto tt, auto dd, auto gg) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    TimedLaunch tl("exact_rows_kernel", st);
    exact_rows_kernel<T, D, G><<<row_blocks(a), kRowWarps * 32, 0, st>>>(static_cast<const T*>(q),
                                                                          static_cast<const T*>(k), a, sel);
    count_launch();
    return cudaGetLastError();
  });
}

}  // namespace pisa
