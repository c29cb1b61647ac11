// Block-sparse attention forward for bf16 prefill (paper §BSA): one warp per
// (kv head, query) row runs MmaAttend over the row's selected leaf blocks.
// Rows are ordered kv-head-major, so consecutive warps read blocks of the
// same head while its keys and values are L2-resident.
#include "attn_mma.cuh"
#include "dispatch.cuh"
#include "kernels.cuh"

namespace pisa {

namespace {

constexpr int kAttnWarps = 4;

template <int D, int CC, int G>
__global__ void __launch_bounds__(kAttnWarps * 32)
    attn_mma_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                    const int32_t* __restrict__ sel, PrefillArgs a, bf16* __restrict__ out, float* __restrict__ lse) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kAttnWarps + warp;
  if (row >= static_cast<int64_t>(a.B) * a.H_kv * a.N) return;
  const int64_t n = a.N;
  const int64_t bh = row / n, t = row % n;
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  const int64_t hs = n * D;
  const int64_t q0 = ((b * a.H_q + h * G) * n + t) * D;
  MmaAttend<D, CC, G> at;
  at.init(q + q0, hs);
  const bf16* kh = k + bh * n * D;
  const bf16* vh = v + bh * n * D;
  const int my = lane < a.K ? sel[row * a.K + lane] : -1;
  for (int x = 0; x < a.K; ++x) {
    const int blk = __shfl_sync(kFull, my, x);
    if (blk >= 0) at.block(kh, vh, static_cast<int64_t>(blk) * CC, n, t, a.causal != 0, a.scale);
  }
  at.store(out + q0, hs, lse ? lse + (b * a.H_q + h * G) * n + t : nullptr, n);
}

}  // namespace

cudaError_t launch_attn_mma(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                            void* out, float* lse, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * a.N;
  const unsigned grid = static_cast<unsigned>((rows + kAttnWarps - 1) / kAttnWarps);
  return dispatch_tdg(PISA_DTYPE_BF16, a.d, a.H_q / a.H_kv, [&](auto, auto dd, auto gg) -> cudaError_t {
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    if (a.C == 64)
      attn_mma_kernel<D, 64, G><<<grid, kAttnWarps * 32, 0, st>>>(
          static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v), sel, a,
          static_cast<bf16*>(out), lse);
    else
      attn_mma_kernel<D, 32, G><<<grid, kAttnWarps * 32, 0, st>>>(
          static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v), sel, a,
          static_cast<bf16*>(out), lse);
    count_launch();
    return cudaGetLastError();
  });
}

}  // namespace pisa
