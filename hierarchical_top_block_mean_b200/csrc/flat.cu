// Flat single-level selection for bf16 queries (paper §BSA: a flat method
// scores all M = ceil(N/C) leaf summaries per query), on tensor cores.
//
// The score u_i = sum_{h'} scale q_{h',t} . kbar_i is linear in q, so the
// group's query heads are summed first (fp32) and the selection is one dense
// contraction [queries x d] . [d x leaves] per kv head. Both operands are
// fp32; each is split into bf16 hi + lo and the product is taken as
// hi.hi + hi.lo + lo.hi (three mma.sync m16n8k16), which reproduces fp32 to
// ~2^-16 relative. The score matrix is never stored: each CTA keeps a running
// top-K per query in shared memory. Candidates are filtered against the
// row's current K-th score (leaves are visited in ascending order, so an
// equal score from a later leaf loses the tie) and inserted by one lane of
// the row's quad at a time.
#include "dispatch.cuh"
#include "kernels.cuh"
#include "mma.cuh"

namespace pisa {

namespace {

constexpr int kFlatWarps = 8;             // 16 queries each: 128 queries per CTA
constexpr int kFlatRows = 16 * kFlatWarps;
constexpr int kChunk = 64;                // leaves per shared-memory chunk

template <int D>
__device__ inline uint2 plane_frag(const bf16* plane, int r, int col) {
  const int ch = col >> 3;
  return *reinterpret_cast<const uint2*>(plane + r * D + ((ch ^ ((r & 3) << 1)) << 3) + (col & 7));
}

template <int D, int G>
__global__ void __launch_bounds__(kFlatWarps * 32, 2)
    flat_mma_kernel(const bf16* __restrict__ q, const float* __restrict__ pyr, int64_t R, PrefillArgs a,
                    int32_t* __restrict__ sel) {
  constexpr int kKS = D / 16;
  extern __shared__ __align__(128) unsigned char smem[];
  float* stage = reinterpret_cast<float*>(smem);                       // [kChunk][D] fp32
  bf16* phi = reinterpret_cast<bf16*>(stage + kChunk * D);             // [kChunk][D] swizzled
  bf16* plo = phi + kChunk * D;                                        // [kChunk][D] swizzled
  float* ls = reinterpret_cast<float*>(plo + kChunk * D);              // [kFlatRows][K]
  int* li = reinterpret_cast<int*>(ls + kFlatRows * kMaxK);            // [kFlatRows][K]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int K = a.K;
  const bool causal = a.causal != 0;
  const int64_t n = a.N;
  const int bh = blockIdx.y;
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  // Longest (latest) query tiles first.
  const int64_t t0 = static_cast<int64_t>(gridDim.x - 1 - blockIdx.x) * kFlatRows;
  const int64_t M1 = level_size(n, a.C, 1);
  const int64_t t_last = min(t0 + kFlatRows - 1, n - 1);
  const int64_t nleaf = causal ? min(M1, t_last / a.C + 1) : M1;
  const float* leaves = pyr + static_cast<int64_t>(bh) * R * D;  // level 1: rows [0, M1)

  for (int x = threadIdx.x; x < kFlatRows * kMaxK; x += blockDim.x) {
    ls[x] = -INFINITY;
    li[x] = INT_MAX;
  }
  auto stage_chunk = [&](int64_t c0) {
    const int64_t cnt = min(static_cast<int64_t>(kChunk), nleaf - c0);
    for (int x = threadIdx.x; x < kChunk * D / 4; x += blockDim.x) {
      const int r = x / (D / 4);
      cp_async16(stage + x * 4, leaves + (r < cnt ? (c0 + r) * D + (x % (D / 4)) * 4 : 0), r < cnt ? 16 : 0);
    }
    cp_async_commit();
  };
  stage_chunk(0);

  // Group sum of the query heads for this lane's rows (gid, gid + 8), split
  // into hi/lo A fragments (four contiguous d columns per lane per k step).
  uint32_t ahi[kKS][4], alo[kKS][4];
  int64_t trow[2];
  bool rok[2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    trow[half] = t0 + 16 * warp + gid + 8 * half;
    rok[half] = trow[half] < n;
    const int64_t tq = rok[half] ? trow[half] : 0;
    const bf16* qp = q + ((b * a.H_q + h * G) * n + tq) * D + 4 * tig;
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 v = load4(qp + static_cast<int64_t>(g) * n * D + 16 * ks);
        s4[0] += v.x;
        s4[1] += v.y;
        s4[2] += v.z;
        s4[3] += v.w;
      }
      float hh[4], ll[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) split_bf16(s4[j], hh[j], ll[j]);
      ahi[ks][half] = pack_bf16(hh[0], hh[1]);
      ahi[ks][2 + half] = pack_bf16(hh[2], hh[3]);
      alo[ks][half] = pack_bf16(ll[0], ll[1]);
      alo[ks][2 + half] = pack_bf16(ll[2], ll[3]);
    }
  }
  // Usable leaves of this lane's two rows (causal: first key <= t).
  int64_t lim[2];
#pragma unroll
  for (int half = 0; half < 2; ++half) lim[half] = causal ? min(nleaf, trow[half] / a.C + 1) : nleaf;
  float thr[2] = {-INFINITY, -INFINITY};
  int thri[2] = {INT_MAX, INT_MAX};
  const int lr0 = 16 * warp + gid;

  for (int64_t c0 = 0; c0 < nleaf; c0 += kChunk) {
    cp_async_wait<0>();
    __syncthreads();
    // fp32 staging -> swizzled bf16 hi / lo planes.
    for (int x = threadIdx.x; x < kChunk * D / 8; x += blockDim.x) {
      const int r = x / (D / 8), ch = x % (D / 8);
      const float4 v0 = *reinterpret_cast<const float4*>(stage + r * D + ch * 8);
      const float4 v1 = *reinterpret_cast<const float4*>(stage + r * D + ch * 8 + 4);
      const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      float hh[8], ll[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) split_bf16(f[j], hh[j], ll[j]);
      const int off = r * D + ((ch ^ ((r & 3) << 1)) << 3);
      *reinterpret_cast<uint4*>(phi + off) =
          make_uint4(pack_bf16(hh[0], hh[1]), pack_bf16(hh[2], hh[3]), pack_bf16(hh[4], hh[5]), pack_bf16(hh[6], hh[7]));
      *reinterpret_cast<uint4*>(plo + off) =
          make_uint4(pack_bf16(ll[0], ll[1]), pack_bf16(ll[2], ll[3]), pack_bf16(ll[4], ll[5]), pack_bf16(ll[6], ll[7]));
    }
    __syncthreads();
    if (c0 + kChunk < nleaf) stage_chunk(c0 + kChunk);

    float acc[kChunk / 8][4];
#pragma unroll
    for (int nt = 0; nt < kChunk / 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
#pragma unroll
      for (int nt = 0; nt < kChunk / 8; ++nt) {
        const uint2 bh2 = plane_frag<D>(phi, 8 * nt + gid, 16 * ks + 4 * tig);
        const uint2 bl2 = plane_frag<D>(plo, 8 * nt + gid, 16 * ks + 4 * tig);
        mma_bf16(acc[nt], ahi[ks], bh2.x, bh2.y);
        mma_bf16(acc[nt], ahi[ks], bl2.x, bl2.y);
        mma_bf16(acc[nt], alo[ks], bh2.x, bh2.y);
      }
    }
    // Candidates: usable leaves whose score beats the row's current K-th.
    uint32_t cand = 0;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
      for (int nt = 0; nt < kChunk / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int64_t i = c0 + 8 * nt + 2 * tig + e;
          acc[nt][2 * half + e] *= a.scale;
          if (rok[half] && i < lim[half] && ranks_before(acc[nt][2 * half + e], static_cast<int>(i), thr[half], thri[half]))
            cand |= 1u << (16 * half + 2 * nt + e);
        }
    }
    if (__ballot_sync(kFull, cand != 0) != 0) {
      for (int tt = 0; tt < 4; ++tt) {
        if (tig == tt && cand) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float* rs = ls + (lr0 + 8 * half) * kMaxK;
            int* ri = li + (lr0 + 8 * half) * kMaxK;
#pragma unroll
            for (int nt = 0; nt < kChunk / 8; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                if (!((cand >> (16 * half + 2 * nt + e)) & 1u)) continue;
                const float v = acc[nt][2 * half + e];
                const int i = static_cast<int>(c0 + 8 * nt + 2 * tig + e);
                if (!ranks_before(v, i, rs[K - 1], ri[K - 1])) continue;
                int p = K - 1;
                while (p > 0 && ranks_before(v, i, rs[p - 1], ri[p - 1])) {
                  rs[p] = rs[p - 1];
                  ri[p] = ri[p - 1];
                  --p;
                }
                rs[p] = v;
                ri[p] = i;
              }
          }
        }
        __syncwarp();
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        thr[half] = ls[(lr0 + 8 * half) * kMaxK + K - 1];
        thri[half] = li[(lr0 + 8 * half) * kMaxK + K - 1];
      }
    }
    __syncthreads();  // planes are rewritten by the next chunk
  }
  // Output: each row's kept leaves, ascending, -1 padded.
  for (int rr = 0; rr < 16; ++rr) {
    const int64_t t = t0 + 16 * warp + rr;
    if (t >= n) break;
    int idx = lane < K ? li[(16 * warp + rr) * kMaxK + lane] : INT_MAX;
    warp_sort_asc(idx);
    if (lane < K) sel[(static_cast<int64_t>(bh) * n + t) * K + lane] = idx == INT_MAX ? -1 : idx;
  }
}

}  // namespace

cudaError_t launch_flat_mma(const PrefillArgs& a, const void* q, const float* pyr, int64_t R, int32_t* sel,
                            cudaStream_t st) {
  return dispatch_tdg(PISA_DTYPE_BF16, a.d, a.H_q / a.H_kv, [&](auto, auto dd, auto gg) -> cudaError_t {
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    const size_t smem = static_cast<size_t>(kChunk) * D * 4 + 2 * static_cast<size_t>(kChunk) * D * 2 +
                        static_cast<size_t>(kFlatRows) * kMaxK * 8;
    auto kern = flat_mma_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(static_cast<unsigned>((a.N + kFlatRows - 1) / kFlatRows), a.B * a.H_kv);
    TimedLaunch tl("flat_mma_kernel", st);
    kern<<<grid, kFlatWarps * 32, smem, st>>>(static_cast<const bf16*>(q), pyr, R, a, sel);
    count_launch();
    return cudaGetLastError();
  });
}

}  // namespace pisa
