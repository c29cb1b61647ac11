// Flat single-level selection on the fifth-generation tensor cores, for bf16
// queries with d = 128 (paper §BSA: a flat method scores all M = ceil(N/C)
// leaf summaries per query).
//
// The score u_i = sum_{h'} scale q_{h',t} . kbar_i is linear in q, so the
// group's heads are summed first and each kv head's selection is one dense
// contraction [queries x d] . [d x leaves]. Both factors are fp32 (the head
// sum and the fp32 summaries); flat_prep_kernel splits each into bf16 hi + lo
// once per call, into the workspace, and the product is taken as
// hi.hi + hi.lo + lo.hi, three tcgen05.mma into one fp32 accumulator, which
// reproduces fp32 to ~2^-16 relative.
//
// flat_umma_kernel: one CTA per (kv head, tile of 128 queries); the tile's
// hi and lo rows stay in shared memory as the A operands.
//   warp 16, one lane (loads): the hi and lo planes of each 64-leaf tile by
//     bulk tensor copy into a ring of kFlStages buffers;
//   warp 17, one lane (MMA): per leaf tile, 3 x 8 tcgen05.mma (M = 128
//     queries, N = 64 leaves, K = 16) into a ring of TMEM accumulators, then
//     commits that free the leaf buffer and publish the accumulator;
//   warps 0-15 (epilogue): four warps per TMEM lane quarter, 8 query rows
//     each; a warp walks its rows two at a time (one per half-warp) testing
//     64 leaves per row at once against the row's K-th best, and merges the
//     rare entrants into the row's running top-K list with a half-warp
//     sorted insert.
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

constexpr int kFlEpiWarps = 16;
constexpr int kFlLoadWarp = kFlEpiWarps;
constexpr int kFlMmaWarp = kFlEpiWarps + 1;
constexpr int kFlThreads = 32 * (kFlEpiWarps + 2);
constexpr int kFlStages = 3;                   // leaf tile buffers (hi + lo)
constexpr int kFlAccStages = 4;                // TMEM accumulators of 64 columns
constexpr uint32_t kFlTmemCols = kFlAccStages * 64;
constexpr int kFlQBytes = 128 * 128 * 2;       // 128 queries x 128 bf16, two 64-column halves
constexpr int kFlLeafBytes = 64 * 128 * 2;     // 64 leaves x 128 bf16, two 64-column halves
constexpr int kFlLists = 128 * kMaxK * 8;      // per query: kMaxK (score, leaf) entries
constexpr int kFlStage = kFlEpiWarps * 8 * 64 * 4;   // per epilogue warp: 8 rows x 64 scores
constexpr int kFlSmem = 1024 + 2 * kFlQBytes + kFlStages * 2 * kFlLeafBytes + kFlLists + kFlStage;

// Workspace: q hi, q lo [B H_kv N][128]; leaf hi, leaf lo [B H_kv M1][128] (bf16).
struct FlatWs {
  bf16 *qhi, *qlo, *khi, *klo;
};
inline size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
size_t flat_ws_carve(const PrefillArgs& a, char* base, FlatWs* w) {
  const size_t qrows = static_cast<size_t>(a.B) * a.H_kv * a.N;
  const size_t krows = static_cast<size_t>(a.B) * a.H_kv * level_size(a.N, a.C, 1);
  const size_t qb = al256(qrows * 128 * 2), kb = al256(krows * 128 * 2);
  if (w) {
    w->qhi = reinterpret_cast<bf16*>(base);
    w->qlo = reinterpret_cast<bf16*>(base + qb);
    w->khi = reinterpret_cast<bf16*>(base + 2 * qb);
    w->klo = reinterpret_cast<bf16*>(base + 2 * qb + kb);
  }
  return 2 * qb + 2 * kb;
}

// Splits x into bf16 hi = bf16(x) and lo = bf16(x - hi).
__device__ inline void split2(float x, bf16& hi, bf16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// One thread per 8 columns of a row: rows [0, qrows) are group-summed query
// rows (b, kv head, t); rows [qrows, qrows + krows) are leaf summaries.
template <int G>
__global__ void __launch_bounds__(256) flat_prep_kernel(const bf16* __restrict__ q, const float* __restrict__ pyr,
                                                        int64_t R, PrefillArgs a, FlatWs w, int64_t qrows,
                                                        int64_t krows, int64_t M1) {
  const int64_t total = (qrows + krows) * 16;
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = x >> 4;
    const int c = static_cast<int>(x & 15) * 8;
    float v[8];
    bf16* dh;
    bf16* dl;
    if (r < qrows) {
      const int64_t bh = r / a.N, t = r % a.N;
      const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint4 u = *reinterpret_cast<const uint4*>(q + ((b * a.H_q + h * G + g) * a.N + t) * 128 + c);
        const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[2 * i] += __uint_as_float(ww[i] << 16);
          v[2 * i + 1] += __uint_as_float(ww[i] & 0xffff0000u);
        }
      }
      dh = w.qhi + r * 128 + c;
      dl = w.qlo + r * 128 + c;
    } else {
      const int64_t kr = r - qrows;
      const int64_t bh = kr / M1, i = kr % M1;
      const float* src = pyr + (bh * R + i) * 128 + c;
      const float4 x0 = *reinterpret_cast<const float4*>(src);
      const float4 x1 = *reinterpret_cast<const float4*>(src + 4);
      v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
      v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
      dh = w.khi + kr * 128 + c;
      dl = w.klo + kr * 128 + c;
    }
    __align__(16) bf16 hh[8], ll[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split2(v[e], hh[e], ll[e]);
    *reinterpret_cast<uint4*>(dh) = *reinterpret_cast<const uint4*>(hh);
    *reinterpret_cast<uint4*>(dl) = *reinterpret_cast<const uint4*>(ll);
  }
}

__global__ void __launch_bounds__(kFlThreads, 1)
    flat_umma_kernel(const __grid_constant__ CUtensorMap tqh, const __grid_constant__ CUtensorMap tql,
                     const __grid_constant__ CUtensorMap tkh, const __grid_constant__ CUtensorMap tkl, PrefillArgs a,
                     int64_t M1, int32_t* __restrict__ sel, unsigned long long* faults) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t qfull, lfull[kFlStages], lempty[kFlStages], accfull[kFlAccStages], accempty[kFlAccStages];
  __shared__ uint32_t tmem_base_sh;
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* qhi = smem;                         // A operands, resident
  unsigned char* qlo = smem + kFlQBytes;
  unsigned char* lbuf = smem + 2 * kFlQBytes;        // [kFlStages][hi, lo][kFlLeafBytes]
  float* ls = reinterpret_cast<float*>(lbuf + kFlStages * 2 * kFlLeafBytes);  // [128][kMaxK] kept scores
  int* li = reinterpret_cast<int*>(ls + 128 * kMaxK);                          // [128][kMaxK] kept leaves
  float* stage_buf = reinterpret_cast<float*>(li + 128 * kMaxK);              // [16 warps][8][64] scores

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool causal = a.causal != 0;
  const int64_t N = a.N;
  const int64_t bh = blockIdx.y;
  const int tile = causal ? static_cast<int>(gridDim.x - 1 - blockIdx.x) : static_cast<int>(blockIdx.x);
  const int64_t t0 = static_cast<int64_t>(tile) * 128;
  const int64_t t_last = (t0 + 127 < N - 1) ? t0 + 127 : N - 1;
  const int64_t nleaf = causal ? (t_last / a.C + 1 < M1 ? t_last / a.C + 1 : M1) : M1;
  const int ntiles = static_cast<int>((nleaf + 63) / 64);

  if (threadIdx.x == 0) {
    mbar_init(&qfull, 1);
    for (int i = 0; i < kFlStages; ++i) {
      mbar_init(&lfull[i], 1);
      mbar_init(&lempty[i], 1);
    }
    for (int i = 0; i < kFlAccStages; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], kFlEpiWarps);
    }
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kFlTmemCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < 128 * kMaxK; i += blockDim.x) {
    ls[i] = -INFINITY;
    li[i] = INT_MAX;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kFlLoadWarp) {
    // ---------------------------------------------------------- loads
    if (lane == 0) {
      const int qy = static_cast<int>(bh * N + t0);
      mbar_expect_tx(&qfull, 2 * kFlQBytes);
      tma_load_2d(qhi, &tqh, 0, qy, &qfull);
      tma_load_2d(qhi + kFlQBytes / 2, &tqh, 64, qy, &qfull);
      tma_load_2d(qlo, &tql, 0, qy, &qfull);
      tma_load_2d(qlo + kFlQBytes / 2, &tql, 64, qy, &qfull);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kFlStages;
        mbar_wait(&lempty[s], ((i / kFlStages) & 1) ^ 1, faults);
        const int ly = static_cast<int>(bh * M1 + static_cast<int64_t>(i) * 64);
        unsigned char* dst = lbuf + s * 2 * kFlLeafBytes;
        mbar_expect_tx(&lfull[s], 2 * kFlLeafBytes);
        tma_load_2d(dst, &tkh, 0, ly, &lfull[s]);
        tma_load_2d(dst + kFlLeafBytes / 2, &tkh, 64, ly, &lfull[s]);
        tma_load_2d(dst + kFlLeafBytes, &tkl, 0, ly, &lfull[s]);
        tma_load_2d(dst + kFlLeafBytes + kFlLeafBytes / 2, &tkl, 64, ly, &lfull[s]);
      }
    }
  } else if (warp == kFlMmaWarp) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      mbar_wait(&qfull, 0, faults);
      const uint32_t ah = smem_u32(qhi), al = smem_u32(qlo);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kFlStages, as = i % kFlAccStages;
        mbar_wait(&lfull[s], (i / kFlStages) & 1, faults);
        mbar_wait(&accempty[as], ((i / kFlAccStages) & 1) ^ 1, faults);
        tc_fence_after();
        const uint32_t bhi = smem_u32(lbuf + s * 2 * kFlLeafBytes), blo = bhi + kFlLeafBytes;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t qo = (ks >> 2) * (kFlQBytes / 2) + (ks & 3) * 32;
          const uint32_t lo = (ks >> 2) * (kFlLeafBytes / 2) + (ks & 3) * 32;
          const uint32_t d = tmem + as * 64;
          umma_bf16(d, sw128_desc(ah + qo), sw128_desc(bhi + lo), kIdesc, ks > 0);
          umma_bf16(d, sw128_desc(ah + qo), sw128_desc(blo + lo), kIdesc, 1);
          umma_bf16(d, sw128_desc(al + qo), sw128_desc(bhi + lo), kIdesc, 1);
        }
        umma_commit(&lempty[s]);
        umma_commit(&accfull[as]);
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // Warp w reads TMEM lane quarter w & 3 and owns 8 of its query rows
    // (part w >> 2). Its lanes stage those rows' 64 scaled scores in shared
    // memory; the warp then walks its rows two at a time, one per half-warp,
    // each lane testing four leaves against the row's K-th best (a ballot
    // skips row pairs with no new entrant, the usual case). A row's running
    // top-K list lives in shared memory, one entry per lane of its half when
    // it changes; entrants are merged one at a time by a half-warp sorted
    // insert, both halves in step. Ranking is by score, then lower leaf
    // index, a total order, so the kept set does not depend on the order in
    // which entrants arrive.
    const int qtr = warp & 3, part = warp >> 2;
    const int row0 = 32 * qtr + 8 * part;  // this warp's rows row0 .. row0 + 7
    const int K = a.K;
    const int half = lane >> 4, hl = lane & 15;
    const unsigned hmask = half ? 0xffff0000u : 0x0000ffffu;
    float* stg = stage_buf + warp * (8 * 64);  // [8 rows][64 leaves] scaled scores
    // Lane r < 8 keeps row row0 + r's K-th best (thr, thri) and usable-leaf limit.
    float thr = -INFINITY;
    int thri = INT_MAX;
    int lim = 0;
    if (lane < 8) {
      const int64_t t = t0 + row0 + lane;
      lim = static_cast<int>(t >= N ? 0 : (causal ? (t / a.C + 1 < M1 ? t / a.C + 1 : M1) : M1));
    }
    for (int i = 0; i < ntiles; ++i) {
      const int as = i % kFlAccStages;
      mbar_wait(&accfull[as], (i / kFlAccStages) & 1, faults);
      __syncwarp();  // the TMEM loads below are warp-collective
      tc_fence_after();
      uint32_t v[64];
      tmem_ld_cols<64>(tmem + (static_cast<uint32_t>(32 * qtr) << 16) + as * 64, v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[as]);
      if ((lane >> 3) == part) {
        float* dst = stg + (lane & 7) * 64;
#pragma unroll
        for (int j = 0; j < 64; j += 4)
          *reinterpret_cast<float4*>(dst + j) =
              make_float4(__uint_as_float(v[j]) * a.scale, __uint_as_float(v[j + 1]) * a.scale,
                          __uint_as_float(v[j + 2]) * a.scale, __uint_as_float(v[j + 3]) * a.scale);
      }
      __syncwarp();
      const int c0 = i * 64;
      for (int rp = 0; rp < 4; ++rp) {
        const int rr = 2 * rp + half;  // this half's row
        const float4 x4 = *reinterpret_cast<const float4*>(stg + rr * 64 + 4 * hl);
        const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
        float th = __shfl_sync(kFull, thr, rr);
        int thi = __shfl_sync(kFull, thri, rr);
        const int lm = __shfl_sync(kFull, lim, rr);
        const int col0 = c0 + 4 * hl;
        unsigned mine = 0;  // this lane's entrants, bit e = leaf col0 + e
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (col0 + e < lm && ranks_before(xv[e], col0 + e, th, thi)) mine |= 1u << e;
        if (__ballot_sync(kFull, mine != 0u) == 0u) continue;
        const int row = row0 + rr;
        float es = hl < K ? ls[row * kMaxK + hl] : -INFINITY;
        int ei = hl < K ? li[row * kMaxK + hl] : INT_MAX;
        for (;;) {
          const unsigned any = __ballot_sync(kFull, mine != 0u);
          if (any == 0u) break;
          const unsigned hany = any & hmask;
          const bool act = hany != 0u;                // this half still has an entrant
          const int src = act ? __ffs(hany) - 1 : lane;  // its lowest lane
          const int e = __ffs(mine | 16u) - 1;         // this lane's lowest entrant (4: none)
          const float my_s = e == 0 ? xv[0] : (e == 1 ? xv[1] : (e == 2 ? xv[2] : xv[3]));
          const float cs = __shfl_sync(kFull, my_s, src);
          const int ci = __shfl_sync(kFull, col0 + e, src);
          if (lane == src && act) mine &= mine - 1u;
          const bool live = act && ranks_before(cs, ci, th, thi);  // the list may have moved past it
          const bool before = live && hl < K && ranks_before(cs, ci, es, ei);
          const float ps = __shfl_up_sync(kFull, es, 1, 16);
          const int pi = __shfl_up_sync(kFull, ei, 1, 16);
          const bool pbefore = __shfl_up_sync(kFull, before, 1, 16) && hl > 0;
          if (before) {
            es = pbefore ? ps : cs;
            ei = pbefore ? pi : ci;
          }
          th = __shfl_sync(kFull, es, K - 1, 16);
          thi = __shfl_sync(kFull, ei, K - 1, 16);
        }
        if (hl < K) {
          ls[row * kMaxK + hl] = es;
          li[row * kMaxK + hl] = ei;
        }
        // Lane r (< 8) takes row r's new threshold from the half that owns it.
        const float th_r = __shfl_sync(kFull, th, (lane & 1) << 4);
        const int thi_r = __shfl_sync(kFull, thi, (lane & 1) << 4);
        if (lane < 8 && (lane >> 1) == rp) {
          thr = th_r;
          thri = thi_r;
        }
      }
    }
    // Kept leaves ascending, -1 padded.
    for (int rr = 0; rr < 8; ++rr) {
      const int row = row0 + rr;
      const int64_t t = t0 + row;
      if (t >= N) break;
      int idx = lane < K ? li[row * kMaxK + lane] : INT_MAX;
      warp_sort_asc(idx);
      if (lane < K) sel[(bh * N + t) * K + lane] = idx == INT_MAX ? -1 : idx;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kFlTmemCols);
  }
}

int flat_sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

bool flat_umma_supported(const PrefillArgs& a) {
  return a.dtype == PISA_DTYPE_BF16 && a.d == 128 &&
         static_cast<int64_t>(a.B) * a.H_kv * a.N + 128 < (int64_t{1} << 31);
}

size_t flat_umma_workspace_bytes(const PrefillArgs& a) {
  return flat_umma_supported(a) ? flat_ws_carve(a, nullptr, nullptr) : 0;
}

cudaError_t launch_flat_umma(const PrefillArgs& a, const void* q, const float* pyr, int64_t R, int32_t* sel, void* ws,
                             cudaStream_t st) {
  FlatWs w;
  flat_ws_carve(a, static_cast<char*>(ws), &w);
  const int64_t M1 = level_size(a.N, a.C, 1);
  const int64_t qrows = static_cast<int64_t>(a.B) * a.H_kv * a.N;
  const int64_t krows = static_cast<int64_t>(a.B) * a.H_kv * M1;
  cudaError_t e = dispatch_tdg(PISA_DTYPE_BF16, 128, a.H_q / a.H_kv, [&](auto, auto, auto gg) -> cudaError_t {
    constexpr int G = decltype(gg)::value;
    const int64_t total = (qrows + krows) * 16;
    const int64_t blocks = (total + 255) / 256;
    const unsigned grid = static_cast<unsigned>(blocks < flat_sm_count() * 32 ? blocks : flat_sm_count() * 32);
    {
      TimedLaunch tl("flat_prep_kernel", st);
      flat_prep_kernel<G><<<grid, 256, 0, st>>>(static_cast<const bf16*>(q), pyr, R, a, w, qrows, krows, M1);
    }
    count_launch();
    return cudaGetLastError();
  });
  if (e != cudaSuccess) return e;
  CUtensorMap tqh, tql, tkh, tkl;
  if ((e = make_tmap_bf16_2d(&tqh, w.qhi, 128, static_cast<uint64_t>(qrows), 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&tql, w.qlo, 128, static_cast<uint64_t>(qrows), 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&tkh, w.khi, 128, static_cast<uint64_t>(krows), 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&tkl, w.klo, 128, static_cast<uint64_t>(krows), 64)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(flat_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFlSmem)) !=
      cudaSuccess)
    return e;
  dim3 grid(static_cast<unsigned>((a.N + 127) / 128), static_cast<unsigned>(a.B * a.H_kv));
  {
    TimedLaunch tl("flat_umma_kernel", st);
    flat_umma_kernel<<<grid, kFlThreads, kFlSmem, st>>>(tqh, tql, tkh, tkl, a, M1, sel, wait_fault_counter());
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace pisa
