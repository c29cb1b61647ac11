// Shared device helpers for the PISA sm_100a kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cfloat>
#include <climits>

#include "../../include/pisa.h"

namespace pisa {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxLevels = 40;  // enough for any N < 2^31 with C >= 1
constexpr int kMaxG = 8;        // query heads per kv head handled by the kernels
constexpr int kMaxK = 16;       // top-K budget; 2K candidates fit one warp

using bf16 = __nv_bfloat16;

// ------------------------------------------------------------ host counter
void count_launch(int n = 1);

// ---------------------------------------------------- per-kernel timing
// Between pisa_timing_start() and pisa_timing_stop() every launch site
// brackets its kernel with two CUDA events recorded on the launching stream:
// a TimedLaunch is constructed just before the launch and destroyed just
// after it. Outside that window construction and destruction do nothing.
class TimedLaunch {
 public:
  TimedLaunch(const char* name, cudaStream_t st);
  ~TimedLaunch();
  TimedLaunch(const TimedLaunch&) = delete;
  TimedLaunch& operator=(const TimedLaunch&) = delete;

 private:
  int slot_;
  cudaStream_t st_;
};

// ----------------------------------------------------------------- geometry
// Pyramid level sizes (paper §Pyramid): M_1 = ceil(n / C), M_{l+1} =
// ceil(M_l / 2). Because ceil(ceil(x / a) / b) = ceil(x / (a b)) for positive
// integers, M_l = ceil(n / (C 2^(l-1))).
// log2 of a power of two.
__host__ __device__ inline int ilog2_pow2(int x) {
#ifdef __CUDA_ARCH__
  return __ffs(x) - 1;
#else
  return __builtin_ctz(static_cast<unsigned>(x));
#endif
}
__host__ __device__ inline bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

__host__ __device__ inline int64_t level_size(int64_t n, int C, int l) {
  if (is_pow2(C)) {  // every block size the kernels support: a shift, not a 64-bit division
    const int sh = ilog2_pow2(C) + l - 1;
    return (n + (int64_t{1} << sh) - 1) >> sh;
  }
  int64_t span = static_cast<int64_t>(C) << (l - 1);
  return (n + span - 1) / span;
}
__host__ __device__ inline int num_levels(int64_t n, int C) {
  int64_t m = (n + C - 1) / C;
  int L = 1;
  while (m > 1) {
    m = (m + 1) / 2;
    ++L;
  }
  return L;
}
// Keys spanned by a nominal block of level l >= 1.
__host__ __device__ inline int64_t level_span(int C, int l) { return static_cast<int64_t>(C) << (l - 1); }

// Row offsets of each level inside one head's pyramid, for a layout sized for
// `n_layout` tokens: level l occupies rows [off[l], off[l] + M_l). Passed to
// kernels by value.
struct Layout {
  int L;                    // levels for n_layout tokens
  int64_t R;                // rows per head
  int64_t off[kMaxLevels + 2];
};
inline Layout make_layout(int64_t n_layout, int C) {
  Layout lay{};
  lay.L = num_levels(n_layout, C);
  int64_t acc = 0;
  for (int l = 1; l <= lay.L; ++l) {
    lay.off[l] = acc;
    acc += level_size(n_layout, C, l);
  }
  lay.off[lay.L + 1] = acc;
  lay.R = acc;
  return lay;
}

// Number of blocks of level l usable by the query at position t (causal
// reading: first key <= t) among the M_l blocks of an n-token sequence.
__device__ inline int64_t valid_count(int64_t n, int C, int l, int64_t t, bool causal) {
  int64_t m = level_size(n, C, l);
  if (!causal) return m;
  int64_t v = (is_pow2(C) ? (t >> (ilog2_pow2(C) + l - 1)) : t / level_span(C, l)) + 1;
  return v < m ? v : m;
}

// --------------------------------------------------------------- loads
__device__ inline float to_f(float x) { return x; }
__device__ inline float to_f(bf16 x) { return __bfloat162float(x); }

// Four consecutive elements starting at p (8-byte aligned for bf16, 16 for fp32).
__device__ inline float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ inline float4 load4(const bf16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float4 f;
  f.x = __uint_as_float(u.x << 16);
  f.y = __uint_as_float(u.x & 0xffff0000u);
  f.z = __uint_as_float(u.y << 16);
  f.w = __uint_as_float(u.y & 0xffff0000u);
  return f;
}
__device__ inline float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}
__device__ inline void store_out(float* p, float v) { *p = v; }
__device__ inline void store_out(bf16* p, float v) { *p = __float2bfloat16_rn(v); }

// --------------------------------------------------------------- warp ops
__device__ inline float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ inline float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Ranking used by every top-K: higher score first, equal scores to the lower
// block index. Empty lanes carry (-inf, INT_MAX) and sort last.
__device__ inline bool ranks_before(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

// Bitonic sort of one (score, index) pair per lane across the warp; lane 0
// ends with the best pair.
__device__ inline void warp_sort_desc(float& s, int& i) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      float os = __shfl_xor_sync(kFull, s, j);
      int oi = __shfl_xor_sync(kFull, i, j);
      bool keep_best = (((lane & k) == 0) == ((lane & j) == 0));
      bool other_first = ranks_before(os, oi, s, i);
      bool mine_first = ranks_before(s, i, os, oi);
      if ((keep_best && other_first) || (!keep_best && mine_first)) {
        s = os;
        i = oi;
      }
    }
  }
}

// Bitonic sort of one index per lane, ascending (INT_MAX = empty, last).
__device__ inline void warp_sort_asc(int& i) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      int oi = __shfl_xor_sync(kFull, i, j);
      bool keep_small = (((lane & k) == 0) == ((lane & j) == 0));
      if (keep_small ? (oi < i) : (oi > i)) i = oi;
    }
  }
}

// Moves the lanes whose flag is set to lanes 0..n-1, keeping their order.
// Returns n. `tmp` is 32 ints of per-warp shared memory.
__device__ inline int warp_compact(int& v, bool keep, int* tmp) {
  const int lane = threadIdx.x & 31;
  unsigned m = __ballot_sync(kFull, keep);
  int pos = __popc(m & ((1u << lane) - 1u));
  __syncwarp();
  if (keep) tmp[pos] = v;
  __syncwarp();
  int n = __popc(m);
  v = lane < n ? tmp[lane] : -1;
  __syncwarp();
  return n;
}

}  // namespace pisa
