// Warp-level tensor-core helpers (mma.sync m16n8k16, bf16 in, fp32 accumulate)
// and the operand layouts the kernels use.
//
// Fragment ownership for lane = 4 * gid + tig (gid = lane / 4, tig = lane % 4):
//   A (16 x 16):  rows gid and gid + 8; k-slots {2 tig, 2 tig + 1} and {2 tig + 8, 2 tig + 9}
//   B (16 x 8):   column gid; k-slots {2 tig, 2 tig + 1} and {2 tig + 8, 2 tig + 9}
//   C (16 x 8):   rows gid and gid + 8; columns 2 tig and 2 tig + 1
// A dot product does not care in which order it visits k, so every kernel maps
// the four k-slots a lane owns in one 16-wide k step to four *contiguous*
// columns 16 ks + 4 tig .. + 3 of the operand rows, for A and B alike. A lane
// then reads its share of a row with one 8-byte (bf16) or 16-byte (fp32) load.
#pragma once

#include "common.cuh"

namespace pisa {

__device__ inline void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ inline uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Splits x into bf16 hi + bf16 lo with x - hi - lo below 2^-16 |x|: the sum of
// two bf16 MMAs against an exact bf16 operand reproduces an fp32 operand.
__device__ inline void split_bf16(float x, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  lo = x - hi;
}

// A-operand registers for rows (r0, r1) from four contiguous fp32 values of
// each row, as hi and lo bf16 parts.
__device__ inline void a_split(const float4& x0, const float4& x1, uint32_t (&hi)[4], uint32_t (&lo)[4]) {
  float h[8], l[8];
  split_bf16(x0.x, h[0], l[0]);
  split_bf16(x0.y, h[1], l[1]);
  split_bf16(x0.z, h[2], l[2]);
  split_bf16(x0.w, h[3], l[3]);
  split_bf16(x1.x, h[4], l[4]);
  split_bf16(x1.y, h[5], l[5]);
  split_bf16(x1.z, h[6], l[6]);
  split_bf16(x1.w, h[7], l[7]);
  hi[0] = pack_bf16(h[0], h[1]);
  hi[1] = pack_bf16(h[4], h[5]);
  hi[2] = pack_bf16(h[2], h[3]);
  hi[3] = pack_bf16(h[6], h[7]);
  lo[0] = pack_bf16(l[0], l[1]);
  lo[1] = pack_bf16(l[4], l[5]);
  lo[2] = pack_bf16(l[2], l[3]);
  lo[3] = pack_bf16(l[6], l[7]);
}

// 16-byte async copy global -> shared; src_bytes < 16 zero-fills the rest.
__device__ inline void cp_async16(void* smem, const void* gmem, int src_bytes) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes));
}
__device__ inline void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ inline void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

}  // namespace pisa
