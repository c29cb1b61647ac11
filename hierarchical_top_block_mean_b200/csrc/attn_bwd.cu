// Backward of the block-sparse attention (paper §BSA) over a fixed selection,
// for bf16 inputs: the selection is a discrete choice, so only the attention
// over the selected blocks' keys is differentiated. For a row (kv head h,
// query t) and query head h' of the group, over the usable keys j:
//   P_j = exp(scale q.k_j - lse),  dP_j = dout . v_j,  D = dout . out,
//   dS_j = P_j (dP_j - D),
//   dq = scale sum_j dS_j k_j,  dk_j += scale dS_j q,  dv_j += P_j dout.
// lse and out are the forward's outputs.
//
// Kernels:
//   bwd_prep_kernel     D per (b, h', t), and the count of rows selecting
//                       each (b, h, leaf);
//   bwd_scan_kernel     one CTA: offsets of the per-leaf query lists and of
//                       the work items (kBwdPairs queries of one leaf);
//   bwd_scatter_kernel  the per-leaf query lists (the selection, inverted);
//   bwd_itemize_kernel  the work-item records;
//   bwd_dq_kernel       one warp per (kv head, query) row at a time, the
//                       row's blocks streamed through a per-warp TMA ring in
//                       16-key chunks (as the forward kernel): S^T = K Q^T,
//                       dP^T = V dO^T, dS, then dQ^T += K^T dS^T;
//   bwd_dkdv_kernel     per work item, the leaf's K and V tiles stay in shared
//                       memory while its queries pass in tiles of 16
//                       (query, head) rows: S = Q K^T and dP = dO V^T split
//                       over the warps by 8-key column tile, P and dS through
//                       shared memory, then dV^T += dO^T P and
//                       dK^T += Q^T dS split by 16-wide d tile; the item's
//                       partial dK, dV are added to the fp32 outputs with
//                       atomics (a leaf's queries may span several items).
// Gradients are fp32. The order in which items add into dk and dv is not
// fixed, so those two are reproducible only up to fp32 rounding.
#include "dispatch.cuh"
#include "kernels.cuh"
#include "mma.cuh"
#include "tma.cuh"
#include "attn_mma.cuh"

namespace pisa {

namespace {

constexpr int kBwdPairs = 64;        // queries per dK/dV work item
constexpr int kDqWarps = 12;
constexpr int kDqKeys = 16;          // keys per streamed chunk
constexpr int kDkvWarps = 8;

// ------------------------------------------------------------------ prep
// D[b, h', t] = dout . out over d (fp32), one warp per (b, h', t).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const bf16* __restrict__ dout, const bf16* __restrict__ out,
                                                       float* __restrict__ Dv, int64_t nrows) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= nrows) return;
  float acc = 0.f;
  for (int e = lane * 4; e < D; e += 128) {
    const float4 g = load4(dout + row * D + e), o = load4(out + row * D + e);
    acc += g.x * o.x + g.y * o.y + g.z * o.z + g.w * o.w;
  }
  acc = warp_sum(acc);
  if (lane == 0) Dv[row] = acc;
}

__global__ void __launch_bounds__(256) bwd_count_kernel(const int32_t* __restrict__ sel, int64_t entries, int K,
                                                        int N, int M1, int32_t* __restrict__ count) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < entries;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int blk = sel[i];
    if (blk < 0 || blk >= M1) continue;
    const int64_t bh = i / (static_cast<int64_t>(N) * K);
    atomicAdd(&count[bh * M1 + blk], 1);
  }
}

// Exclusive scans of the list lengths and of the work items per list.
__global__ void __launch_bounds__(1024) bwd_scan_kernel(const int32_t* __restrict__ count, int nb,
                                                        int32_t* __restrict__ off, int32_t* __restrict__ item_off) {
  __shared__ int wsum[2][32];
  __shared__ int carry[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  for (int base = 0; base < nb; base += 4096) {
    int c[4], it[4], s0 = 0, s1 = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = base + threadIdx.x * 4 + j;
      c[j] = i < nb ? count[i] : 0;
      it[j] = (c[j] + kBwdPairs - 1) / kBwdPairs;
      s0 += c[j];
      s1 += it[j];
    }
    int x0 = s0, x1 = s1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y0 = __shfl_up_sync(kFull, x0, o), y1 = __shfl_up_sync(kFull, x1, o);
      if (lane >= o) {
        x0 += y0;
        x1 += y1;
      }
    }
    if (lane == 31) {
      wsum[0][warp] = x0;
      wsum[1][warp] = x1;
    }
    __syncthreads();
    if (warp == 0) {
      int w0 = wsum[0][lane], w1 = wsum[1][lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y0 = __shfl_up_sync(kFull, w0, o), y1 = __shfl_up_sync(kFull, w1, o);
        if (lane >= o) {
          w0 += y0;
          w1 += y1;
        }
      }
      wsum[0][lane] = w0;
      wsum[1][lane] = w1;
    }
    __syncthreads();
    int e0 = carry[0] + (warp ? wsum[0][warp - 1] : 0) + x0 - s0;
    int e1 = carry[1] + (warp ? wsum[1][warp - 1] : 0) + x1 - s1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = base + threadIdx.x * 4 + j;
      if (i < nb) {
        off[i] = e0;
        item_off[i] = e1;
      }
      e0 += c[j];
      e1 += it[j];
    }
    __syncthreads();
    if (threadIdx.x == 1023) {
      carry[0] = e0;
      carry[1] = e1;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    off[nb] = carry[0];
    item_off[nb] = carry[1];
  }
}

__global__ void __launch_bounds__(256) bwd_scatter_kernel(const int32_t* __restrict__ sel, int64_t entries, int K,
                                                          int N, int M1, const int32_t* __restrict__ off,
                                                          int32_t* __restrict__ fill, int32_t* __restrict__ qlist) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < entries;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int blk = sel[i];
    if (blk < 0 || blk >= M1) continue;
    const int64_t row = i / K;
    const int64_t bh = row / N;
    const int t = static_cast<int>(row % N);
    const int64_t b = bh * M1 + blk;
    qlist[off[b] + atomicAdd(&fill[b], 1)] = t;
  }
}

__global__ void __launch_bounds__(256) bwd_itemize_kernel(const int32_t* __restrict__ off,
                                                          const int32_t* __restrict__ item_off, int nb, int M1,
                                                          int4* __restrict__ items) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nb) return;
  const int bh = b / M1, leaf = b % M1;
  for (int i = item_off[b]; i < item_off[b + 1]; ++i) {
    const int lo = off[b] + (i - item_off[b]) * kBwdPairs;
    items[i] = make_int4(bh, lo, min(lo + kBwdPairs, off[b + 1]), leaf);
  }
}

// ------------------------------------------------------------------ dQ
struct DqCursor {
  int64_t row;   // -1: exhausted
  int bh, t;     // row = bh * N + t
  int blk_lane;  // this lane's entry of the row's compacted block list
  int nblk, idx, half;
};

template <int D, int CC, int G>
__global__ void __launch_bounds__(kDqWarps * 32, 1)
    bwd_dq_kernel(const bf16* __restrict__ q, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const int32_t* __restrict__ sel,
                  const bf16* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ Dv,
                  PrefillArgs a, float* __restrict__ dq, unsigned long long* faults) {
  constexpr int kKS = D / 16;
  constexpr int kChunkBytes = kDqKeys * D * 2;
  constexpr int kHalves = CC / kDqKeys;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t bars[kDqWarps][2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem + warp * (2 * 2 * kChunkBytes);  // [stage][K|V][chunk]
  if (lane == 0) {
    mbar_init(&bars[warp][0], 1);
    mbar_init(&bars[warp][1], 1);
    mbar_init_fence();
  }
  __syncwarp();
  uint32_t phase = 0;
  const int64_t n = a.N;
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * n;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kDqWarps;
  const bool causal = a.causal != 0;

  auto load_row = [&](int64_t r) -> DqCursor {
    for (; r < rows; r += stride) {
      int b = lane < a.K ? sel[r * a.K + lane] : -1;
      const unsigned m = __ballot_sync(kFull, b >= 0);
      if (m == 0) continue;
      int out_b = b;
      if ((m & (m + 1u)) != 0u) {  // not a prefix: compact, lane j takes the j-th valid entry
        out_b = -1;
        for (int j = 0, src = 0; j < 32; ++j) {
          const int bj = __shfl_sync(kFull, b, j);
          if ((m >> j) & 1u) {
            if (lane == src) out_b = bj;
            ++src;
          }
        }
      }
      return DqCursor{r, static_cast<int>(r / n), static_cast<int>(r % n), out_b, __popc(m), 0, 0};
    }
    return DqCursor{-1, 0, 0, -1, 0, 0, 0};
  };
  auto advance = [&](const DqCursor& c) -> DqCursor {
    if (c.row < 0) return c;
    if (c.half + 1 < kHalves) return DqCursor{c.row, c.bh, c.t, c.blk_lane, c.nblk, c.idx, c.half + 1};
    if (c.idx + 1 < c.nblk) return DqCursor{c.row, c.bh, c.t, c.blk_lane, c.nblk, c.idx + 1, 0};
    return load_row(c.row + stride);
  };
  auto issue = [&](const DqCursor& c, int st) {
    if (c.row < 0) return;
    const int blk = __shfl_sync(kFull, c.blk_lane, c.idx);
    if (lane == 0) {
      const int y = static_cast<int>(c.bh * n + static_cast<int64_t>(blk) * CC + c.half * kDqKeys);
      unsigned char* ks = ring + st * 2 * kChunkBytes;
      unsigned char* vs = ks + kChunkBytes;
      fence_proxy_async();
      mbar_expect_tx(&bars[warp][st], 2 * kChunkBytes);
#pragma unroll
      for (int x = 0; x < D; x += 64) {
        tma_load_2d(ks + x * kDqKeys * 2, &tmk, x, y, &bars[warp][st]);
        tma_load_2d(vs + x * kDqKeys * 2, &tmv, x, y, &bars[warp][st]);
      }
    }
  };

  DqCursor cur = load_row(static_cast<int64_t>(blockIdx.x) * kDqWarps + warp);
  issue(cur, 0);
  int st = 0;
  int64_t row_now = -1;
  int hb = 0, hh = 0;
  uint32_t qb[kKS][2], gb[kKS][2];
  float ls[2], dd[2], acc[kKS][4];

  while (cur.row >= 0) {
    const DqCursor nxt = advance(cur);
    issue(nxt, st ^ 1);
    mbar_wait(&bars[warp][st], (phase >> st) & 1u, faults);
    phase ^= 1u << st;

    const int t = cur.t;
    if (cur.row != row_now) {  // first chunk of a row: q, dout, lse, D
      row_now = cur.row;
      hb = cur.bh / a.H_kv;
      hh = cur.bh % a.H_kv;
      const int64_t qrow = (static_cast<int64_t>(hb) * a.H_q + hh * G + (gid < G ? gid : 0)) * n + t;
      const bf16* qp = q + qrow * D + 2 * tig;
      const bf16* gp = dout + qrow * D + 2 * tig;
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks) {
        qb[ks][0] = gid < G ? *reinterpret_cast<const uint32_t*>(qp + 16 * ks) : 0u;
        qb[ks][1] = gid < G ? *reinterpret_cast<const uint32_t*>(qp + 16 * ks + 8) : 0u;
        gb[ks][0] = gid < G ? *reinterpret_cast<const uint32_t*>(gp + 16 * ks) : 0u;
        gb[ks][1] = gid < G ? *reinterpret_cast<const uint32_t*>(gp + 16 * ks + 8) : 0u;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int hd = 2 * tig + j;
        const int64_t lrow = (static_cast<int64_t>(hb) * a.H_q + hh * G + (hd < G ? hd : 0)) * n + t;
        ls[j] = hd < G ? lse[lrow] : 0.f;
        dd[j] = hd < G ? Dv[lrow] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kKS; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    }
    const int last = (causal && t < n - 1) ? t : static_cast<int>(n - 1);
    const int blk = __shfl_sync(kFull, cur.blk_lane, cur.idx);
    const int key0 = blk * CC + cur.half * kDqKeys;
    const unsigned char* ks_ = ring + st * 2 * kChunkBytes;
    const unsigned char* vs_ = ks_ + kChunkBytes;

    // S^T = K Q^T and dP^T = V dO^T (16 keys x 8 heads each).
    float s[4] = {0.f, 0.f, 0.f, 0.f}, dp[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int mat = lane >> 3, r = lane & 7;
      const int krow = r + 8 * (mat & 1);
#pragma unroll
      for (int kk = 0; kk < kKS; ++kk) {
        uint32_t af[4], vf[4];
        ldsm_x4(af, ks_ + swz128<kDqKeys>(krow, 8 * (2 * kk + (mat >> 1))));
        ldsm_x4(vf, vs_ + swz128<kDqKeys>(krow, 8 * (2 * kk + (mat >> 1))));
        mma_bf16(s, af, qb[kk][0], qb[kk][1]);
        mma_bf16(dp, vf, gb[kk][0], gb[kk][1]);
      }
    }
    // P and dS (rows: keys gid, gid + 8; columns: heads 2 tig, 2 tig + 1).
    float ds[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = i & 1;
      const bool ok = key0 + gid + 8 * (i >> 1) <= last;
      const float p = ok ? expf(s[i] * a.scale - ls[j]) : 0.f;
      ds[i] = p * (dp[i] - dd[j]);
    }
    const uint32_t db0 = movtrans(pack_bf16(ds[0], ds[1])), db1 = movtrans(pack_bf16(ds[2], ds[3]));
    // dQ^T (d x heads) += K^T dS^T.
    {
      const int mat = lane >> 3, r = lane & 7;
      const int krow = r + 8 * (mat >> 1);
#pragma unroll
      for (int md = 0; md < kKS; ++md) {
        uint32_t af[4];
        ldsm_x4_t(af, ks_ + swz128<kDqKeys>(krow, 8 * (2 * md + (mat & 1))));
        mma_bf16(acc[md], af, db0, db1);
      }
    }
    __syncwarp();  // this stage is refilled by the next iteration's prefetch

    if (nxt.row != cur.row) {  // last chunk of the row: write scale * dQ
      const int64_t hs = n * D;
      float* o0 = dq + ((static_cast<int64_t>(hb) * a.H_q + hh * G) * n + t) * D;
#pragma unroll
      for (int md = 0; md < kKS; ++md)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int d = 16 * md + gid + 8 * rr;
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (2 * tig + j < G) o0[(2 * tig + j) * hs + d] = a.scale * acc[md][2 * rr + j];
        }
    }
    cur = nxt;
    st ^= 1;
  }
}

// ------------------------------------------------------------------ dK, dV
// Byte offset of element (row, col) in a row-major bf16 tile of kCols
// columns whose 16-byte chunks are swizzled by row (chunk c of row r at
// c ^ (r & m), m = min(chunks per row, 8) - 1), so ldmatrix reads of 8 rows
// spread over the bank groups.
template <int kCols>
__device__ inline uint32_t tsw(int row, int col) {
  constexpr int kMask = (kCols / 8 >= 8 ? 8 : kCols / 8) - 1;
  return static_cast<uint32_t>(row * kCols * 2 + (((col >> 3) ^ (row & kMask)) << 4) + ((col & 7) << 1));
}

template <int D, int CC, int G>
struct DkvSmem {
  static constexpr int kRows = 16;                        // (query, head) rows per query tile
  static constexpr int kK = 0;                            // K tile [CC][D]
  static constexpr int kV = kK + CC * D * 2;              // V tile [CC][D]
  static constexpr int kQ = kV + CC * D * 2;              // Q rows [2][16][D] (double buffered)
  static constexpr int kG = kQ + 2 * kRows * D * 2;       // dout rows [2][16][D]
  static constexpr int kP = kG + 2 * kRows * D * 2;       // P [16][CC]
  static constexpr int kS = kP + kRows * CC * 2;          // dS [16][CC]
  static constexpr int kL = kS + kRows * CC * 2;          // lse [2][16]
  static constexpr int kDD = kL + 2 * kRows * 4;          // D [2][16]
  static constexpr int kT = kDD + 2 * kRows * 4;          // query position per row [2][16]
  static constexpr int kTq = kT + 2 * kRows * 4;          // the item's query positions [kBwdPairs]
  static constexpr int kBytes = kTq + kBwdPairs * 4 + 128;
};

// 4-byte asynchronous copy global -> shared; src_bytes = 0 writes zero.
__device__ inline void cp_async4(void* smem, const void* gmem, int src_bytes) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes));
}

template <int D, int CC, int G>
__global__ void __launch_bounds__(kDkvWarps * 32)
    bwd_dkdv_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                    const bf16* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ Dv,
                    const int4* __restrict__ items, const int32_t* __restrict__ item_total,
                    const int32_t* __restrict__ qlist, PrefillArgs a, float* __restrict__ dk,
                    float* __restrict__ dv) {
  using SM = DkvSmem<D, CC, G>;
  constexpr int kQT = 16 / G;       // queries per tile
  constexpr int kNT = CC / 8;       // 8-key column tiles
  constexpr int kKS = D / 16;       // k steps over d (phase A); d tiles (phase B)
  extern __shared__ __align__(128) unsigned char sm[];
  unsigned char* Ks = sm + SM::kK;
  unsigned char* Vs = sm + SM::kV;
  unsigned char* Qs = sm + SM::kQ;
  unsigned char* Gs = sm + SM::kG;
  unsigned char* Ps = sm + SM::kP;
  unsigned char* Ss = sm + SM::kS;
  float* Ls = reinterpret_cast<float*>(sm + SM::kL);
  float* DDs = reinterpret_cast<float*>(sm + SM::kDD);
  int* Ts = reinterpret_cast<int*>(sm + SM::kT);
  int* Tq = reinterpret_cast<int*>(sm + SM::kTq);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t n = a.N;
  const bool causal = a.causal != 0;
  const int total = *item_total;

  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    const int4 it = items[item];
    const int64_t bh = it.x;
    const int blk = it.w;
    const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
    const int key_base = blk * CC;
    const int nkeys = static_cast<int>(min(static_cast<int64_t>(CC), n - key_base));
    const int npairs = it.z - it.y;
    const int ntiles = (npairs + kQT - 1) / kQT;
    if (threadIdx.x < kBwdPairs) Tq[threadIdx.x] = threadIdx.x < npairs ? qlist[it.y + threadIdx.x] : -1;
    // The leaf's K and V rows (zero past the sequence).
    for (int i = threadIdx.x; i < CC * (D / 8); i += blockDim.x) {
      const int r = i / (D / 8), c = (i % (D / 8)) * 8;
      const bool ok = r < nkeys;
      const int64_t src = (bh * n + key_base + (ok ? r : 0)) * D + c;
      cp_async16(Ks + tsw<D>(r, c), k + src, ok ? 16 : 0);
      cp_async16(Vs + tsw<D>(r, c), v + src, ok ? 16 : 0);
    }
    cp_async_commit();
    __syncthreads();  // Tq
    // Query tile i -> buffer f: rows r = (query qi, head g), qi = r / G.
    auto issue = [&](int i, int f) {
      for (int x = threadIdx.x; x < 16 * (D / 8); x += blockDim.x) {
        const int r = x / (D / 8), c = (x % (D / 8)) * 8;
        const int t = Tq[i * kQT + r / G];
        const int64_t src = ((b * a.H_q + h * G + r % G) * n + (t >= 0 ? t : 0)) * D + c;
        cp_async16(Qs + f * (16 * D * 2) + tsw<D>(r, c), q + src, t >= 0 ? 16 : 0);
        cp_async16(Gs + f * (16 * D * 2) + tsw<D>(r, c), dout + src, t >= 0 ? 16 : 0);
      }
      if (threadIdx.x < 16) {
        const int r = threadIdx.x;
        const int t = Tq[i * kQT + r / G];
        const int64_t lrow = (b * a.H_q + h * G + r % G) * n + (t >= 0 ? t : 0);
        cp_async4(Ls + 16 * f + r, lse + lrow, t >= 0 ? 4 : 0);
        cp_async4(DDs + 16 * f + r, Dv + lrow, t >= 0 ? 4 : 0);
        Ts[16 * f + r] = t;
      }
    };
    issue(0, 0);
    cp_async_commit();
    float dka[kNT][4], dva[kNT][4];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) dka[nt][i] = dva[nt][i] = 0.f;

    for (int i = 0; i < ntiles; ++i) {
      const int f = i & 1;
      if (i + 1 < ntiles) issue(i + 1, f ^ 1);
      cp_async_commit();
      cp_async_wait<1>();  // K, V and tile i have landed
      __syncthreads();
      const unsigned char* Qf = Qs + f * (16 * D * 2);
      const unsigned char* Gf = Gs + f * (16 * D * 2);

      // Phase A: warp w < kNT takes keys [8 w, 8 w + 8): S = Q K^T and
      // dP = dO V^T over d, then P and dS into shared memory.
      if (warp < kNT) {
        float s[4] = {0.f, 0.f, 0.f, 0.f}, dp[4] = {0.f, 0.f, 0.f, 0.f};
        const int mi = lane >> 3;
        const int arow = (lane & 7) + 8 * (mi & 1);
        const int krow = 8 * warp + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < kKS; ks += 2) {
          uint32_t bk[4], bv[4];
          ldsm_x4(bk, Ks + tsw<D>(krow, 16 * ks + 8 * mi));
          ldsm_x4(bv, Vs + tsw<D>(krow, 16 * ks + 8 * mi));
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            uint32_t aq[4], ag[4];
            ldsm_x4(aq, Qf + tsw<D>(arow, 16 * (ks + u) + 8 * (mi >> 1)));
            ldsm_x4(ag, Gf + tsw<D>(arow, 16 * (ks + u) + 8 * (mi >> 1)));
            mma_bf16(s, aq, bk[2 * u], bk[2 * u + 1]);
            mma_bf16(dp, ag, bv[2 * u], bv[2 * u + 1]);
          }
        }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int r = gid + 8 * rr;
          const int t = Ts[16 * f + r];
          const float l = Ls[16 * f + r], dd = DDs[16 * f + r];
          float pv[2], sv[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int key = 8 * warp + 2 * tig + j;
            const bool ok = t >= 0 && key < nkeys && (!causal || key_base + key <= t);
            const float p = ok ? expf(s[2 * rr + j] * a.scale - l) : 0.f;
            pv[j] = p;
            sv[j] = p * (dp[2 * rr + j] - dd);
          }
          *reinterpret_cast<uint32_t*>(Ps + tsw<CC>(r, 8 * warp + 2 * tig)) = pack_bf16(pv[0], pv[1]);
          *reinterpret_cast<uint32_t*>(Ss + tsw<CC>(r, 8 * warp + 2 * tig)) = pack_bf16(sv[0], sv[1]);
        }
      }
      __syncthreads();

      // Phase B: warp w < kKS takes d rows [16 w, 16 w + 16):
      // dV^T += dO^T P and dK^T += Q^T dS over the tile's 16 rows.
      if (warp < kKS) {
        const int mi = lane >> 3;
        uint32_t ag[4], aq[4];
        {
          const int r = (lane & 7) + 8 * (mi >> 1);
          ldsm_x4_t(ag, Gf + tsw<D>(r, 16 * warp + 8 * (mi & 1)));
          ldsm_x4_t(aq, Qf + tsw<D>(r, 16 * warp + 8 * (mi & 1)));
        }
        const int brow = (lane & 7) + 8 * (mi & 1);
#pragma unroll
        for (int nt = 0; nt < kNT; nt += 2) {
          uint32_t bp[4], bs[4];
          ldsm_x4_t(bp, Ps + tsw<CC>(brow, 8 * (nt + (mi >> 1))));
          ldsm_x4_t(bs, Ss + tsw<CC>(brow, 8 * (nt + (mi >> 1))));
          mma_bf16(dva[nt], ag, bp[0], bp[1]);
          mma_bf16(dka[nt], aq, bs[0], bs[1]);
          if (nt + 1 < kNT) {
            mma_bf16(dva[nt + 1], ag, bp[2], bp[3]);
            mma_bf16(dka[nt + 1], aq, bs[2], bs[3]);
          }
        }
      }
      __syncthreads();  // P, dS and this buffer are rewritten two steps on
    }
    cp_async_wait<0>();
    // The item's partial gradients: dV^T, dK^T rows d = 16 w + gid (+8),
    // columns keys 8 nt + 2 tig (+1).
    if (warp < kKS) {
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int d = 16 * warp + gid + 8 * (i >> 1);
          const int key = 8 * nt + 2 * tig + (i & 1);
          if (key < nkeys) {
            const int64_t o = (bh * n + key_base + key) * D + d;
            atomicAdd(dv + o, dva[nt][i]);
            atomicAdd(dk + o, a.scale * dka[nt][i]);
          }
        }
    }
    __syncthreads();  // K, V and Tq are reloaded for the next item
  }
}

int sm_count_bwd() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

inline size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct BwdWs {
  float* D;
  int32_t *count, *fill, *off, *item_off, *qlist;
  int4* items;
};

size_t carve_bwd(const PrefillArgs& a, char* base, BwdWs* w) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * a.N;
  const int64_t nb = static_cast<int64_t>(a.B) * a.H_kv * level_size(a.N, a.C, 1);
  const int64_t pairs = rows * a.K;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + o : nullptr;
    o += al256(bytes);
    return p;
  };
  BwdWs x;
  x.D = reinterpret_cast<float*>(take(static_cast<size_t>(a.B) * a.H_q * a.N * 4));
  x.count = reinterpret_cast<int32_t*>(take(nb * 4));
  x.fill = reinterpret_cast<int32_t*>(take(nb * 4));
  x.off = reinterpret_cast<int32_t*>(take((nb + 1) * 4));
  x.item_off = reinterpret_cast<int32_t*>(take((nb + 1) * 4));
  x.qlist = reinterpret_cast<int32_t*>(take(pairs * 4));
  x.items = reinterpret_cast<int4*>(take((pairs / kBwdPairs + nb + 1) * 16));
  if (w) *w = x;
  return o;
}

}  // namespace

size_t attn_bwd_workspace_bytes(const PrefillArgs& a) { return carve_bwd(a, nullptr, nullptr); }

cudaError_t launch_attn_bwd(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                            const void* out, const float* lse, const void* dout, float* dq, float* dk, float* dv,
                            void* ws, cudaStream_t st) {
  BwdWs w;
  carve_bwd(a, static_cast<char*>(ws), &w);
  const int M1 = static_cast<int>(level_size(a.N, a.C, 1));
  const int nb = a.B * a.H_kv * M1;
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * a.N;
  const int64_t entries = rows * a.K;
  const int64_t qrows = static_cast<int64_t>(a.B) * a.H_q * a.N;
  const int G = a.H_q / a.H_kv;
  cudaError_t e;
  if ((e = cudaMemsetAsync(w.count, 0, static_cast<size_t>(nb) * 4, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(w.fill, 0, static_cast<size_t>(nb) * 4, st)) != cudaSuccess) return e;
  const size_t kv_bytes = static_cast<size_t>(rows) * a.d * 4;
  // Rows that select no block keep dq = 0.
  if ((e = cudaMemsetAsync(dq, 0, static_cast<size_t>(qrows) * a.d * 4, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dk, 0, kv_bytes, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dv, 0, kv_bytes, st)) != cudaSuccess) return e;
  const int64_t eblocks = (entries + 255) / 256;
  const unsigned eg = static_cast<unsigned>(eblocks < 148 * 64 ? eblocks : 148 * 64);
  e = dispatch_td(PISA_DTYPE_BF16, a.d, [&](auto, auto dd) -> cudaError_t {
    constexpr int D = decltype(dd)::value;
    TimedLaunch tl("bwd_prep_kernel", st);
    bwd_prep_kernel<D><<<static_cast<unsigned>((qrows * 32 + 255) / 256), 256, 0, st>>>(
        static_cast<const bf16*>(dout), static_cast<const bf16*>(out), w.D, qrows);
    count_launch();
    return cudaGetLastError();
  });
  if (e != cudaSuccess) return e;
  {
    TimedLaunch tl("bwd_count_kernel", st);
    bwd_count_kernel<<<eg, 256, 0, st>>>(sel, entries, a.K, a.N, M1, w.count);
  }
  count_launch();
  {
    TimedLaunch tl("bwd_scan_kernel", st);
    bwd_scan_kernel<<<1, 1024, 0, st>>>(w.count, nb, w.off, w.item_off);
  }
  count_launch();
  {
    TimedLaunch tl("bwd_scatter_kernel", st);
    bwd_scatter_kernel<<<eg, 256, 0, st>>>(sel, entries, a.K, a.N, M1, w.off, w.fill, w.qlist);
  }
  count_launch();
  {
    TimedLaunch tl("bwd_itemize_kernel", st);
    bwd_itemize_kernel<<<static_cast<unsigned>((nb + 255) / 256), 256, 0, st>>>(w.off, w.item_off, nb, M1, w.items);
  }
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  CUtensorMap tmk, tmv;
  if ((e = make_tmap_bf16_2d(&tmk, k, a.d, static_cast<uint64_t>(rows), kDqKeys)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&tmv, v, a.d, static_cast<uint64_t>(rows), kDqKeys)) != cudaSuccess) return e;
  unsigned long long* faults = wait_fault_counter();
  const int64_t want = (rows + kDqWarps - 1) / kDqWarps;
  const unsigned grid = static_cast<unsigned>(want < sm_count_bwd() ? want : sm_count_bwd());
  return dispatch_tdg(PISA_DTYPE_BF16, a.d, G, [&](auto, auto dd, auto gg) -> cudaError_t {
    constexpr int D = decltype(dd)::value, GG = decltype(gg)::value;
    const size_t smem_dq = static_cast<size_t>(kDqWarps) * 2 * 2 * kDqKeys * D * 2 + 1024;
    auto kq = a.C == 64 ? bwd_dq_kernel<D, 64, GG> : bwd_dq_kernel<D, 32, GG>;
    cudaError_t e2 = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_dq));
    if (e2 != cudaSuccess) return e2;
    {
      TimedLaunch tl("bwd_dq_kernel", st);
      kq<<<grid, kDqWarps * 32, smem_dq, st>>>(static_cast<const bf16*>(q), tmk, tmv, sel,
                                              static_cast<const bf16*>(dout), lse, w.D, a, dq, faults);
    }
    count_launch();
    if ((e2 = cudaGetLastError()) != cudaSuccess) return e2;
    const int smem_kv = a.C == 64 ? DkvSmem<D, 64, GG>::kBytes : DkvSmem<D, 32, GG>::kBytes;
    auto kk = a.C == 64 ? bwd_dkdv_kernel<D, 64, GG> : bwd_dkdv_kernel<D, 32, GG>;
    e2 = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv);
    if (e2 != cudaSuccess) return e2;
    int per_sm = 0;
    e2 = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kk, kDkvWarps * 32, smem_kv);
    if (e2 != cudaSuccess) return e2;
    TimedLaunch tl("bwd_dkdv_kernel", st);
    kk<<<static_cast<unsigned>(sm_count_bwd() * (per_sm > 0 ? per_sm : 1)), kDkvWarps * 32, smem_kv, st>>>(
        static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v),
        static_cast<const bf16*>(dout), lse, w.D, w.items, w.item_off + nb, w.qlist, a, dk, dv);
    count_launch();
    return cudaGetLastError();
  });
}

}  // namespace pisa
