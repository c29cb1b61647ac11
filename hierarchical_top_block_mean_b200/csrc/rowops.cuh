// Warp-per-row device routines: fused coarse-to-fine selection for one
// (kv head, query) row, block-sparse attention for one row, and the running
// top-K merge used by the flat selector.
//
// One warp owns one row. The routine keeps the (at most 2K <= 32) candidates
// of a level one per lane, so every per-level step (validity filter, keep-all
// rule, top-K, expansion to children) is a handful of warp shuffles.
#pragma once

#include "common.cuh"

namespace pisa {

// log(exp(a) + exp(b)) for a finite a and b (b may be -inf).
__device__ inline float lse2(float a, float b) {
  const float m = fmaxf(a, b);
  return m + logf(expf(a - m) + expf(b - m));
}

// Bitonic sort of (index, payload) pairs ascending by index (INT_MAX last).
__device__ inline void warp_sort_asc_kv(int& i, float& s) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      int oi = __shfl_xor_sync(kFull, i, j);
      float os = __shfl_xor_sync(kFull, s, j);
      bool keep_small = (((lane & k) == 0) == ((lane & j) == 0));
      if (keep_small ? (oi < i) : (oi > i)) {
        i = oi;
        s = os;
      }
    }
  }
}

// Merges a chunk of (score, index) pairs (one per lane, any order) into the
// running best list held sorted in lanes 0..31 (best first). Afterwards the
// lanes hold the 32 best of both, sorted.
__device__ inline void warp_merge_best(float& bs, int& bi, float s, int i) {
  const int lane = threadIdx.x & 31;
  warp_sort_desc(s, i);
  // Best-first list against the reversed chunk: the better of each pair
  // forms a bitonic sequence holding the 32 best of the union.
  float rs = __shfl_sync(kFull, s, 31 - lane);
  int ri = __shfl_sync(kFull, i, 31 - lane);
  if (ranks_before(rs, ri, bs, bi)) {
    bs = rs;
    bi = ri;
  }
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    float os = __shfl_xor_sync(kFull, bs, j);
    int oi = __shfl_xor_sync(kFull, bi, j);
    bool lower = (lane & j) == 0;
    if (lower ? ranks_before(os, oi, bs, bi) : ranks_before(bs, bi, os, oi)) {
      bs = os;
      bi = oi;
    }
  }
}

// Everything one row's selection needs.
template <typename T, int D, int G>
struct SelectRow {
  const float* q;    // shared memory, [G][D] fp32 query heads of the group
  const float* pyr;  // this head's pyramid, rows of D fp32
  const int64_t* off;  // off[l] = first row of level l (layout of the pyramid)
  const T* k;        // this head's raw keys, rows of D
  int64_t n;         // tokens held
  int64_t t;         // query position
  int C, K;
  bool causal;
  float scale;
  int* tmp;          // 32 ints of per-warp shared memory

  __device__ bool usable(int l, int64_t i) const {
    if (i < 0 || i >= level_size(n, C, l)) return false;
    return !causal || i * level_span(C, l) <= t;
  }

  // Score of candidate block c of level l >= 2: sum over the group of the
  // LSE over its (one or two) usable child summaries (paper §TopK, §Kernels).
  __device__ float inner_score(int l, int64_t c) const {
    const int64_t r0 = 2 * c;
    const bool has1 = usable(l - 1, r0 + 1);
    const float* row0 = pyr + (off[l - 1] + r0) * D;
    float a0[G], a1[G];
#pragma unroll
    for (int g = 0; g < G; ++g) a0[g] = a1[g] = 0.f;
#pragma unroll 4
    for (int e = 0; e < D; e += 4) {
      const float4 x0 = load4(row0 + e);
      const float4 x1 = has1 ? load4(row0 + D + e) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 qq = *reinterpret_cast<const float4*>(q + g * D + e);
        a0[g] += dot4(qq, x0);
        a1[g] += dot4(qq, x1);
      }
    }
    float u = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) u += has1 ? lse2(scale * a0[g], scale * a1[g]) : scale * a0[g];
    return u;
  }

  // Exact raw-key LSE of leaf block c, summed over the group; computed by the
  // whole warp (lanes over keys). Returns the same value in every lane.
  __device__ float leaf_score(int64_t c) const {
    const int lane = threadIdx.x & 31;
    float acc[2][G];
    bool ok[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t j = c * C + lane + 32 * h;
      ok[h] = (lane + 32 * h < C) && j < n && (!causal || j <= t);
#pragma unroll
      for (int g = 0; g < G; ++g) acc[h][g] = 0.f;
      if (ok[h]) {
        const T* kr = k + j * D;
#pragma unroll 4
        for (int e = 0; e < D; e += 4) {
          const float4 x = load4(kr + e);
#pragma unroll
          for (int g = 0; g < G; ++g) acc[h][g] += dot4(*reinterpret_cast<const float4*>(q + g * D + e), x);
        }
      }
    }
    float u = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float s0 = ok[0] ? scale * acc[0][g] : -INFINITY;
      const float s1 = ok[1] ? scale * acc[1][g] : -INFINITY;
      const float m = warp_max(fmaxf(s0, s1));
      const float z = warp_sum((ok[0] ? expf(s0 - m) : 0.f) + (ok[1] ? expf(s1 - m) : 0.f));
      u += m + logf(z);
    }
    return u;
  }

  // Coarse-to-fine selection (paper §TopK). Starts at the highest level that
  // has more than K usable blocks, with all of them as candidates; every
  // level above it keeps all its usable blocks unscored, so this equals
  // starting from the root. Returns the kept leaves in lanes 0..nk-1 (sorted
  // ascending) with their leaf scores (NaN when kept unscored).
  __device__ int run(int& leaf, float& score) const {
    const int lane = threadIdx.x & 31;
    const int L = num_levels(n, C);
    int l = L;
    while (l >= 1 && valid_count(n, C, l, t, causal) <= K) --l;
    if (l < 1) {  // even the leaf level has <= K usable blocks: keep them all
      const int nv = static_cast<int>(valid_count(n, C, 1, t, causal));
      leaf = lane < nv ? lane : -1;
      score = __int_as_float(0x7fffffff);
      return nv;
    }
    int cand = lane < valid_count(n, C, l, t, causal) ? lane : -1;
    int nk = 0;
    float s = -INFINITY;
    for (;; --l) {
      const int nc = warp_compact(cand, cand >= 0 && usable(l, cand), tmp);
      if (nc <= K) {
        nk = nc;
        s = __int_as_float(0x7fffffff);
      } else {
        if (l >= 2) {
          s = lane < nc ? inner_score(l, cand) : -INFINITY;
        } else {
          s = -INFINITY;
          for (int x = 0; x < nc; ++x) {
            const float u = leaf_score(__shfl_sync(kFull, cand, x));
            if (lane == x) s = u;
          }
        }
        int idx = lane < nc ? cand : INT_MAX;
        warp_sort_desc(s, idx);
        cand = idx;
        nk = K;
      }
      if (l == 1) break;
      const int parent = __shfl_sync(kFull, cand, lane >> 1);
      cand = (lane >> 1) < nk ? 2 * parent + (lane & 1) : -1;
    }
    int idx = lane < nk ? cand : INT_MAX;
    float sc = lane < nk ? s : 0.f;
    warp_sort_asc_kv(idx, sc);
    leaf = lane < nk ? idx : -1;
    score = sc;
    return nk;
  }
};

// Online-softmax attention of the G query heads of one row over the raw keys
// of the selected leaf blocks (paper §BSA). Lanes take 32 keys at a time for
// the logits and the output columns for the weighted sum of values.
template <typename T, int D, int G>
struct AttendRow {
  static constexpr int kCols = D / 32;
  const float* q;     // shared [G][D] fp32
  const T* k;         // this head's keys
  const T* v;         // this head's values
  int64_t n, t;
  int C;
  bool causal;
  float scale;
  float* p;           // per-warp shared [G][32]

  __device__ void run(const int* blocks, int nb, float (&o)[G][kCols], float (&m)[G], float (&l)[G]) const {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < kCols; ++e) o[g][e] = 0.f;
    }
    for (int bi = 0; bi < nb; ++bi) {
      const int64_t b = blocks[bi];
      if (b < 0) continue;
      const int64_t hi = (b + 1) * C < n ? (b + 1) * C : n;
      for (int64_t j0 = b * C; j0 < hi; j0 += 32) {
        const int64_t j = j0 + lane;
        const bool ok = j < hi && (!causal || j <= t);
        float s[G];
#pragma unroll
        for (int g = 0; g < G; ++g) s[g] = 0.f;
        if (ok) {
          const T* kr = k + j * D;
#pragma unroll 4
          for (int e = 0; e < D; e += 4) {
            const float4 x = load4(kr + e);
#pragma unroll
            for (int g = 0; g < G; ++g) s[g] += dot4(*reinterpret_cast<const float4*>(q + g * D + e), x);
          }
        }
        const unsigned live = __ballot_sync(kFull, ok);
        if (live == 0) continue;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float x = ok ? scale * s[g] : -INFINITY;
          const float mn = fmaxf(m[g], warp_max(x));
          const float alpha = (m[g] == -INFINITY) ? 0.f : expf(m[g] - mn);
          const float pv = ok ? expf(x - mn) : 0.f;
          l[g] = l[g] * alpha + warp_sum(pv);
#pragma unroll
          for (int e = 0; e < kCols; ++e) o[g][e] *= alpha;
          m[g] = mn;
          p[g * 32 + lane] = pv;
        }
        __syncwarp();
        for (int jj = 0; jj < 32; ++jj) {
          if (!((live >> jj) & 1u)) continue;
          const T* vr = v + (j0 + jj) * D + lane * kCols;
          float vv[kCols];
#pragma unroll
          for (int e = 0; e < kCols; ++e) vv[e] = to_f(vr[e]);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pw = p[g * 32 + jj];
#pragma unroll
            for (int e = 0; e < kCols; ++e) o[g][e] = fmaf(pw, vv[e], o[g][e]);
          }
        }
        __syncwarp();
      }
    }
  }
};


// Stages the G query heads of one row into per-warp shared memory as fp32.
template <typename T, int D, int G>
__device__ inline void stage_q(const T* __restrict__ qrow0, int64_t head_stride, float* qs) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int g = 0; g < G; ++g)
    for (int e = lane * 4; e < D; e += 128) {
      const float4 x = load4(qrow0 + g * head_stride + e);
      *reinterpret_cast<float4*>(qs + g * D + e) = x;
    }
  __syncwarp();
}


}  // namespace pisa
