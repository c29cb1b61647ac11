// Exact-score flat selection: every usable leaf block of the sequence is
// scored by the LSE of its raw keys summed over the GQA group (the leaf-level
// score of the pyramid search, paper §TopK, applied to all blocks as a flat
// method does, §BSA), then the top K per (kv head, query).
//
// tcgen05 kernel for bf16, d = 128, C = 64: one CTA owns a tile of 128 / G_Q
// queries of one kv head, i.e. 128 (query, head) rows, which stay in shared
// memory as the MMA's A operand for the CTA's whole life. The leaves stream
// past it:
//   warp 8, one lane (loads): each leaf's 64 x 128 key tile by bulk tensor
//     copy into a ring of kKStages buffers;
//   warp 9, one lane (MMA): per leaf, eight tcgen05.mma (M = 128 rows,
//     N = 64 keys, K = 16) into a ring of TMEM accumulators, then commits that
//     free the key buffer and publish the accumulator;
//   warps 0-7 (epilogue): warps w and w + 4 share TMEM lane quarter w; each
//     thread owns one lane = one (query, head) row and loads 32 of its 64
//     logits; the two halves' partial max and exp-sum are combined through
//     shared memory into the row's LSE over the usable keys; the G_Q heads of
//     a query are summed by shuffles, and the query's first lane keeps a
//     running top-K list in shared memory (entries are rarely displaced once
//     the list is full, so the insertion sort costs little).
// Causal tiles stop at the last leaf their latest query can use and are
// launched longest first. Every mbarrier wait is bounded in time; the TMEM
// allocation is always released before exit.
#include "dispatch.cuh"
#include "kernels.cuh"
#include "mma.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace pisa {

namespace {

constexpr int kExEpiWarps = 8;              // warps 0-7 epilogue (two per TMEM lane quarter)
constexpr int kExLoadWarp = kExEpiWarps;    // warp 8 loads key tiles
constexpr int kExMmaWarp = kExEpiWarps + 1; // warp 9 issues the MMAs
constexpr int kExThreads = 32 * (kExEpiWarps + 2);
constexpr int kExKStages = 3;               // key tile buffers
constexpr int kExAccStages = 4;             // TMEM accumulators of 64 columns
constexpr uint32_t kExTmemCols = kExAccStages * 64;
constexpr int kExQBytes = 128 * 128 * 2;    // 128 rows x 128 bf16: two 64-column halves
constexpr int kExKeyBytes = 64 * 128 * 2;   // 64 keys x 128 bf16: two 64-column halves

template <int G>
struct ExSmem {
  static constexpr int kQT = 128 / G;  // queries per tile
  static constexpr int kLists = kQT * kMaxK * 8;
  static constexpr int kBytes = 1024 + kExQBytes + kExKStages * kExKeyBytes + kLists;
};

template <int G>
__global__ void __launch_bounds__(kExThreads, 2)
    exact_umma_kernel(const bf16* __restrict__ q, const __grid_constant__ CUtensorMap tmk, PrefillArgs a,
                      int32_t* __restrict__ sel, unsigned long long* faults) {
  constexpr int kQT = ExSmem<G>::kQT;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t kfull[kExKStages], kempty[kExKStages], accfull[kExAccStages], accempty[kExAccStages];
  __shared__ uint32_t tmem_base_sh;
  __shared__ float2 xch[2][4][32];  // per leaf parity and lane quarter: the second half's (max, sum) per row
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* qbuf = smem;               // A operand, resident
  unsigned char* kbuf = smem + kExQBytes;   // [kExKStages][kExKeyBytes]
  float* ls = reinterpret_cast<float*>(kbuf + kExKStages * kExKeyBytes);  // [kQT][kMaxK] kept scores
  int* li = reinterpret_cast<int*>(ls + kQT * kMaxK);                     // [kQT][kMaxK] kept leaves

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool causal = a.causal != 0;
  const int64_t N = a.N;
  const int64_t bh = blockIdx.y;
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  const int tile = causal ? static_cast<int>(gridDim.x - 1 - blockIdx.x) : static_cast<int>(blockIdx.x);
  const int64_t t0 = static_cast<int64_t>(tile) * kQT;
  const int64_t M1 = (N + 63) / 64;
  const int64_t t_last = (t0 + kQT - 1 < N - 1) ? t0 + kQT - 1 : N - 1;
  const int nleaf = static_cast<int>(causal ? (t_last / 64 + 1 < M1 ? t_last / 64 + 1 : M1) : M1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kExKStages; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < kExAccStages; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], kExEpiWarps);
    }
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kExTmemCols);
    tmem_relinquish();
  }
  // The tile's rows (query qi, head g) -> row qi * G + g, 128-byte swizzled
  // K-major halves; rows past the sequence are zero.
  for (int i = threadIdx.x; i < 128 * 16; i += blockDim.x) {
    const int r = i >> 4, c = i & 15;
    const int qi = r / G, g = r % G;
    const int64_t t = t0 + qi;
    const bool ok = t < N;
    const bf16* src = q + ((b * a.H_q + h * G + g) * N + (ok ? t : 0)) * 128 + c * 8;
    cp_async16(qbuf + (c >> 3) * (kExQBytes / 2) + r * 128 + (((c & 7) ^ (r & 7)) << 4), src, ok ? 16 : 0);
  }
  cp_async_commit();
  for (int i = threadIdx.x; i < kQT * kMaxK; i += blockDim.x) {
    ls[i] = -INFINITY;
    li[i] = INT_MAX;
  }
  cp_async_wait<0>();
  fence_proxy_async();  // the tensor cores read what cp.async wrote
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kExLoadWarp) {
    // ---------------------------------------------------------- key loads
    if (lane == 0) {
      for (int i = 0; i < nleaf; ++i) {
        const int s = i % kExKStages;
        mbar_wait(&kempty[s], ((i / kExKStages) & 1) ^ 1, faults);
        const int y = static_cast<int>(bh * N + static_cast<int64_t>(i) * 64);
        mbar_expect_tx(&kfull[s], kExKeyBytes);
        tma_load_2d(kbuf + s * kExKeyBytes, &tmk, 0, y, &kfull[s]);
        tma_load_2d(kbuf + s * kExKeyBytes + 64 * 128, &tmk, 64, y, &kfull[s]);
      }
    }
  } else if (warp == kExMmaWarp) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t qa = smem_u32(qbuf);
      for (int i = 0; i < nleaf; ++i) {
        const int s = i % kExKStages, as = i % kExAccStages;
        mbar_wait(&kfull[s], (i / kExKStages) & 1, faults);
        mbar_wait(&accempty[as], ((i / kExAccStages) & 1) ^ 1, faults);
        tc_fence_after();
        const uint32_t ka = smem_u32(kbuf + s * kExKeyBytes);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t qo = (ks >> 2) * (kExQBytes / 2) + (ks & 3) * 32;
          const uint32_t ko = (ks >> 2) * (64 * 128) + (ks & 3) * 32;
          umma_bf16(tmem + as * 64, sw128_desc(qa + qo), sw128_desc(ka + ko), kIdesc, ks > 0);
        }
        umma_commit(&kempty[s]);
        umma_commit(&accfull[as]);
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int qtr = warp & 3, hf = warp >> 2;  // TMEM lane quarter; half of the 64 key columns
    const int row = 32 * qtr + lane;
    const int qi = row / G;
    const int64_t t = t0 + qi;
    const bool qok = t < N;
    const bool owner = hf == 0 && (row % G) == 0;
    const int K = a.K;
    const float sl2 = a.scale * 1.4426950408889634f;
    float* rs = ls + qi * kMaxK;
    int* ri = li + qi * kMaxK;
    float thr = -INFINITY;
    int thri = INT_MAX;
    for (int i = 0; i < nleaf; ++i) {
      const int as = i % kExAccStages;
      mbar_wait(&accfull[as], (i / kExAccStages) & 1, faults);
      __syncwarp();  // the TMEM load below is warp-collective
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * qtr) << 16) + as * 64 + 32 * hf, v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[as]);
      // Usable keys of leaf i for this query: j < N and, causally, j <= t.
      const int64_t key0 = static_cast<int64_t>(i) * 64;
      int64_t lim = N - key0;
      if (causal && t - key0 + 1 < lim) lim = t - key0 + 1;
      const int nv = qok ? static_cast<int>(lim < 0 ? 0 : (lim > 64 ? 64 : lim)) : 0;
      // This warp's half of the columns: partial max and exp-sum, then the
      // halves of a row are combined through shared memory.
      const int nvh = nv - 32 * hf;
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (nvh >= 32) {
#pragma unroll
        for (int j = 0; j < 32; ++j) m4[j & 3] = fmaxf(m4[j & 3], __uint_as_float(v[j]));
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvh) m4[j & 3] = fmaxf(m4[j & 3], __uint_as_float(v[j]));
      }
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      const float mxs = mx * sl2;
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      if (nvh >= 32) {
#pragma unroll
        for (int j = 0; j < 32; ++j) s4[j & 3] += ex2_approx(fmaf(__uint_as_float(v[j]), sl2, -mxs));
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvh) s4[j & 3] += ex2_approx(fmaf(__uint_as_float(v[j]), sl2, -mxs));
      }
      const float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      const int xb = i & 1;
      if (hf == 1) xch[xb][qtr][lane] = make_float2(mx, sum);
      named_sync(1 + qtr, 64);  // the two warps of this lane quarter
      if (hf == 1) continue;
      float u = 0.f;
      if (nv > 0) {
        const float2 o = xch[xb][qtr][lane];
        const float m = fmaxf(mx, o.x);
        float z = 0.f;
        if (mx != -INFINITY) z += sum * ex2_approx((mx - m) * sl2);
        if (o.x != -INFINITY) z += o.y * ex2_approx((o.x - m) * sl2);
        u = m * a.scale + logf(z);
      }
      // The G rows of a query are G consecutive lanes and share nv.
#pragma unroll
      for (int o = 1; o < G; o <<= 1) u += __shfl_xor_sync(kFull, u, o);
      if (owner && nv > 0 && ranks_before(u, i, thr, thri)) {
        int p = K - 1;
        while (p > 0 && ranks_before(u, i, rs[p - 1], ri[p - 1])) {
          rs[p] = rs[p - 1];
          ri[p] = ri[p - 1];
          --p;
        }
        rs[p] = u;
        ri[p] = i;
        thr = rs[K - 1];
        thri = ri[K - 1];
      }
    }
    if (owner && qok) {
      // Kept leaves ascending, -1 padded.
      for (int m = 1; m < K; ++m) {
        const int x = ri[m];
        int p = m;
        while (p > 0 && ri[p - 1] > x) {
          ri[p] = ri[p - 1];
          --p;
        }
        ri[p] = x;
      }
      int32_t* out = sel + (bh * N + t) * K;
      for (int m = 0; m < K; ++m) out[m] = ri[m] == INT_MAX ? -1 : ri[m];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kExTmemCols);
  }
}

}  // namespace

bool exact_umma_supported(const PrefillArgs& a) {
  const int G = a.H_q / a.H_kv;
  return a.dtype == PISA_DTYPE_BF16 && a.d == 128 && a.C == 64 && (G == 1 || G == 2 || G == 4 || G == 8) &&
         static_cast<int64_t>(a.B) * a.H_kv * a.N + 64 < (int64_t{1} << 31);
}

cudaError_t launch_exact_umma(const PrefillArgs& a, const void* q, const void* k, int32_t* sel, cudaStream_t st) {
  CUtensorMap tmk;
  cudaError_t e = make_tmap_bf16_2d(&tmk, k, 128, static_cast<uint64_t>(a.B) * a.H_kv * a.N, 64);
  if (e != cudaSuccess) return e;
  return dispatch_tdg(PISA_DTYPE_BF16, 128, a.H_q / a.H_kv, [&](auto, auto, auto gg) -> cudaError_t {
    constexpr int G = decltype(gg)::value;
    constexpr int kQT = ExSmem<G>::kQT;
    const int smem = ExSmem<G>::kBytes;
    auto kern = exact_umma_kernel<G>;
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e2 != cudaSuccess) return e2;
    dim3 grid(static_cast<unsigned>((a.N + kQT - 1) / kQT), static_cast<unsigned>(a.B * a.H_kv));
    TimedLaunch tl("exact_umma_kernel", st);
    kern<<<grid, kExThreads, smem, st>>>(static_cast<const bf16*>(q), tmk, a, sel, wait_fault_counter());
    count_launch();
    return cudaGetLastError();
  });
}

}  // namespace pisa
