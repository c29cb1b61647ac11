// Tensor-core block-sparse attention for one (kv head, query) row, computed
// by one warp (paper §BSA): o = sum_j exp(s_j) v_j / sum_j exp(s_j) over the
// raw keys j of the selected leaf blocks, s_j = scale q.k_j, for the G query
// heads of the group at once.
//
// Formulation (per leaf block of CC keys):
//   S^T [CC keys x 8 heads]  = K [CC x D] . Q^T [D x 8]      (A = K, B = Q^T)
//   O^T [D x 8 heads]       += V^T [D x CC] . P^T [CC x 8]   (A = V^T, B = P^T)
// Keys and d sit on the MMA's M dimension and the (at most 8) heads on N, so
// no MMA row is padding when G = 8. K and V are read straight from global
// memory (L2) into registers with 8-byte loads; the two operands that are
// needed transposed (V^T and P^T) are transposed in registers with
// movmatrix, so the kernel needs no shared memory. Online softmax keeps one
// running max and sum per head; each lane owns heads 2 tig and 2 tig + 1.
#pragma once

#include "mma.cuh"

namespace pisa {

__device__ inline uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// d index held by O^T row slot r (0..15) of d-tile md: V is loaded with four
// contiguous columns per lane, which the register transpose turns into this
// slot order.
__device__ inline int od_index(int md, int r) {
  const int g = r & 7;
  return 16 * md + 4 * (g >> 1) + (g & 1) + ((r >> 3) << 1);
}

template <int D, int CC, int G>
struct MmaAttend {
  static constexpr int kKS = D / 16;   // k steps of S^T and d tiles of O^T
  static constexpr int kMT = CC / 16;  // 16-key tiles per block
  static_assert(G >= 1 && G <= 8, "at most 8 heads per group");

  uint32_t qb[kKS][2];  // B fragments of Q^T (heads >= G are zero)
  float m[2], l[2];     // running max / sum for heads 2 tig, 2 tig + 1
  float o[kKS][4];      // O^T accumulators: d tile md, rows (slots) gid / gid + 8, heads 2 tig, 2 tig + 1

  // q0: head 0 of the group at this query; head_stride elements between heads.
  __device__ void init(const bf16* __restrict__ q0, int64_t head_stride) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const bf16* qp = q0 + (gid < G ? gid : 0) * head_stride + 4 * tig;
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
      uint2 u = make_uint2(0u, 0u);
      if (gid < G) u = *reinterpret_cast<const uint2*>(qp + 16 * ks);
      qb[ks][0] = u.x;
      qb[ks][1] = u.y;
    }
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
#pragma unroll
    for (int i = 0; i < kKS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  }

  // Adds the keys [key0, key0 + CC) of one block (rows of kh / vh, D elements
  // each), restricted to key < n and, when causal, key <= t.
  __device__ void block(const bf16* __restrict__ kh, const bf16* __restrict__ vh, int64_t key0, int64_t n,
                        int64_t t, bool causal, float scale) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    int64_t last = n - 1;
    if (causal && t < last) last = t;
    const bool full = key0 + CC - 1 <= last;
    // ---- S^T = K Q^T
    float s[kMT][4];
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
      const int64_t k0 = key0 + 16 * mt + gid;
      const int64_t ka = k0 <= last ? k0 : last;
      const int64_t kb = k0 + 8 <= last ? k0 + 8 : last;
      const bf16* pa = kh + ka * D + 4 * tig;
      const bf16* pb = kh + kb * D + 4 * tig;
      uint2 ua[kKS], ub[kKS];
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks) {
        ua[ks] = __ldg(reinterpret_cast<const uint2*>(pa + 16 * ks));
        ub[ks] = __ldg(reinterpret_cast<const uint2*>(pb + 16 * ks));
      }
      s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks) {
        const uint32_t a[4] = {ua[ks].x, ub[ks].x, ua[ks].y, ub[ks].y};
        mma_bf16(s[mt], a, qb[ks][0], qb[ks][1]);
      }
    }
    // ---- online softmax per head (column); rows of this lane: keys 16 mt + gid (+8)
    float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const bool ok = full || key0 + 16 * mt + gid + 8 * r <= last;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float x = ok ? s[mt][2 * r + j] * scale : -INFINITY;
          s[mt][2 * r + j] = x;
          bm[j] = fmaxf(bm[j], x);
        }
      }
    }
    float alpha[2], mn[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      bm[j] = fmaxf(bm[j], __shfl_xor_sync(kFull, bm[j], 4));
      bm[j] = fmaxf(bm[j], __shfl_xor_sync(kFull, bm[j], 8));
      bm[j] = fmaxf(bm[j], __shfl_xor_sync(kFull, bm[j], 16));
      mn[j] = fmaxf(m[j], bm[j]);
      alpha[j] = (m[j] == -INFINITY) ? 0.f : expf(m[j] - mn[j]);
      m[j] = mn[j];
    }
    float ps[2] = {0.f, 0.f};
    uint32_t pb[kMT][2];
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
      float p[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = i & 1;
        p[i] = (s[mt][i] == -INFINITY) ? 0.f : expf(s[mt][i] - mn[j]);
        ps[j] += p[i];
      }
      // P^T tiles (keys x heads) -> B fragments (heads x keys) by transposition.
      pb[mt][0] = movtrans(pack_bf16(p[0], p[1]));
      pb[mt][1] = movtrans(pack_bf16(p[2], p[3]));
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      ps[j] += __shfl_xor_sync(kFull, ps[j], 4);
      ps[j] += __shfl_xor_sync(kFull, ps[j], 8);
      ps[j] += __shfl_xor_sync(kFull, ps[j], 16);
      l[j] = l[j] * alpha[j] + ps[j];
    }
#pragma unroll
    for (int md = 0; md < kKS; ++md) {
      o[md][0] *= alpha[0];
      o[md][1] *= alpha[1];
      o[md][2] *= alpha[0];
      o[md][3] *= alpha[1];
    }
    // ---- O^T += V^T P^T, one 16-key step at a time
#pragma unroll
    for (int kk = 0; kk < kMT; ++kk) {
      const int64_t k0 = key0 + 16 * kk + gid;
      const int64_t ka = k0 <= last ? k0 : last;
      const int64_t kb = k0 + 8 <= last ? k0 + 8 : last;
      const bf16* pa = vh + ka * D + 4 * tig;
      const bf16* pv = vh + kb * D + 4 * tig;
      uint2 ua[kKS], ub[kKS];
#pragma unroll
      for (int md = 0; md < kKS; ++md) {
        ua[md] = __ldg(reinterpret_cast<const uint2*>(pa + 16 * md));
        ub[md] = __ldg(reinterpret_cast<const uint2*>(pv + 16 * md));
      }
#pragma unroll
      for (int md = 0; md < kKS; ++md) {
        const uint32_t a[4] = {movtrans(ua[md].x), movtrans(ua[md].y), movtrans(ub[md].x), movtrans(ub[md].y)};
        mma_bf16(o[md], a, pb[kk][0], pb[kk][1]);
      }
    }
  }

  // Merges another partial state (same lane mapping) into this one.
  __device__ void merge(const float (&m2)[2], const float (&l2)[2], const float (&o2)[kKS][4]) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float mn = fmaxf(m[j], m2[j]);
      const float a1 = m[j] == -INFINITY ? 0.f : expf(m[j] - mn);
      const float a2 = m2[j] == -INFINITY ? 0.f : expf(m2[j] - mn);
      l[j] = l[j] * a1 + l2[j] * a2;
#pragma unroll
      for (int md = 0; md < kKS; ++md) {
        o[md][j] = o[md][j] * a1 + o2[md][j] * a2;
        o[md][2 + j] = o[md][2 + j] * a1 + o2[md][2 + j] * a2;
      }
      m[j] = mn;
    }
  }

  // Writes o / l for the G heads: out0 = head 0's output row, head_stride
  // elements between heads; lse0 likewise (may be null).
  template <typename TO>
  __device__ void store(TO* __restrict__ out0, int64_t head_stride, float* __restrict__ lse0,
                        int64_t lse_stride) const {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    float inv[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) inv[j] = l[j] > 0.f ? 1.f / l[j] : 0.f;
#pragma unroll
    for (int md = 0; md < kKS; ++md) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int d = od_index(md, gid + 8 * r);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int hd = 2 * tig + j;
          if (hd < G) store_out(out0 + hd * head_stride + d, o[md][2 * r + j] * inv[j]);
        }
      }
    }
    if (lse0 && gid == 0) {
#pragma unroll
      for (int j = 0; j < 2; ++j)
        if (2 * tig + j < G) lse0[(2 * tig + j) * lse_stride] = m[j] + logf(l[j]);
    }
  }
};

}  // namespace pisa
