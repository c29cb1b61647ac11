// Top scored levels of the coarse-to-fine search on tcgen05 tensor cores
// (paper §TopK, the inner-level score; §Kernels, stage 1).
//
// The first scored levels of a query's search are small: the start level has
// at most 2K usable nodes and each level below at most twice as many, and
// the queries of a short run of positions start at the same level. So
// instead of gathering the children of each query's candidates, one CTA
// scores every node of the block's three top levels for 16 consecutive
// queries of one kv head at once: the 128 (query, head) rows are the A
// operand (M = 128), the children summaries of a level the B operand in
// chunks of 64 rows (N = 64), once with their bf16 hi parts and once with
// their lo parts into the same fp32 accumulator (the split reproduces the
// fp32 summary to 2^-16). The epilogue forms each node's score exactly as
// the router does: per head the log-sum-exp of the scaled logits of the
// node's usable children, summed over the G_Q = 8 heads of the group; the
// children usable for a query are those whose first key is at or before it.
//
// Warp roles (576 threads, one persistent CTA per SM):
//   warp 16, one lane: copies. Each block's query tile by a 3-D bulk tensor
//     copy (dimensions d, head, position, so that a query's 8 heads are 8
//     adjacent rows) into one of two tile buffers; the children of each level
//     in chunks of 128 rows (hi and lo parts) by 2-D bulk tensor copies into a
//     ring of two stages;
//   warp 17, one lane: MMAs, 16 per chunk (8 k steps x hi, lo; N = 128). The
//     block's two passes go to two TMEM accumulators: levels Ltop and
//     Ltop - 1 (at most 64 and 128 children) into columns 0..127 and
//     128..255, and Ltop - 2 (at most 256 children) into columns 256..511;
//   warps 0-15: four epilogue groups of four warps: Ltop's nodes, Ltop - 1's
//     nodes (pass 0), and the two halves of Ltop - 2's nodes (pass 1), so
//     that both passes of a block and the next block's MMAs overlap. Thread =
//     TMEM lane = (query, head) row; a node's two children are adjacent
//     columns; the head sum is a butterfly reduce-scatter over the 8 lanes of
//     a query (16 nodes, 14 shuffles), after which each lane stores two
//     nodes' scores.
// Every wait is bounded (kWaitNs), like the other kernels' waits.
#include "dispatch.cuh"
#include "select2_ws.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace pisa {

namespace {

constexpr int kTopEpiWarps = 16;
constexpr int kTopThreads = 32 * (kTopEpiWarps + 2);
constexpr int kTopRows = 128;                        // kDenseQ queries x 8 heads
constexpr int kTopABytes = kTopRows * 128 * 2;       // 32 KB: two 64-column halves of 16 KB
constexpr int kTopChunkRows = 128;                   // children per chunk (MMA N)
constexpr int kTopHalf = kTopChunkRows * 128;        // one 128-row x 64-column half of a chunk part: 16 KB
constexpr int kTopChunkBytes = 4 * kTopHalf;         // hi and lo, two halves each: 64 KB
constexpr int kTopStages = 2;
constexpr int kTopSmem = 1024 + 2 * kTopABytes + kTopStages * kTopChunkBytes;
constexpr uint32_t kTopCols = 512;

// The block's levels: lev[i] = Ltop - i (i < nl), children count nch[i] at
// level lev[i] - 1, node count nn[i] usable by the block's last query.
struct TopGeom {
  int nl;
  int lev[3], nch[3], nn[3];
};

// Level geometry from a shared table of level sizes (C a power of two):
// usable blocks of level l for position t.
struct LevelTab {
  int L, lc;                    // levels, log2 C
  int64_t size[kMaxLevels + 2];  // blocks per level
};
__device__ inline int64_t tab_valid(const LevelTab& T, int l, int64_t t, bool causal) {
  if (!causal) return T.size[l];
  const int64_t v = (t >> (T.lc + l - 1)) + 1;
  return v < T.size[l] ? v : T.size[l];
}
__device__ inline TopGeom top_geom(const LevelTab& T, int K, int64_t t_last, bool causal) {
  TopGeom g{};
  int lt = T.L;
  while (lt >= 1 && tab_valid(T, lt, t_last, causal) <= K) --lt;
  for (int i = 0; i < 3; ++i) {
    const int l = lt - i;
    if (l < 2) break;
    const int64_t vc = tab_valid(T, l, t_last, causal);
    g.lev[g.nl] = l;
    g.nn[g.nl] = static_cast<int>(vc);
    g.nch[g.nl] = static_cast<int>(min(2 * vc, T.size[l - 1]));
    ++g.nl;
  }
  return g;
}
// Children rows of chunk j of a block, rounded up to the MMA's N granule.
__device__ inline int chunk_rows(const TopGeom& g, int j) {
  const int i = j < 2 ? j : 2;
  const int rows = j < 2 ? g.nch[i] : min(g.nch[2] - 128 * (j - 2), 128);
  return min(128, (rows + 15) & ~15);
}
// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, both
// K-major, M = 128, N = n (a multiple of 16, at most 256).
__device__ inline uint32_t idesc_n(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(n) >> 3) << 17) | ((128u >> 4) << 24);
}

// Chunk schedule of a block: chunk 0 = level 0 (<= 64 children), chunk 1 =
// level 1 (<= 128), chunks 2, 3 = level 2 (<= 256). TMEM column of each.
__device__ inline int n_chunks_total(const TopGeom& g) {
  return g.nl < 3 ? g.nl : 2 + (g.nch[2] + kTopChunkRows - 1) / kTopChunkRows;
}
__device__ inline int chunk_level(int j) { return j < 2 ? j : 2; }
__device__ inline int chunk_col(int j) { return j < 2 ? kTopChunkRows * j : 256 + kTopChunkRows * (j - 2); }

// 2^x and log2 x by the hardware's approximate instructions (errors near
// 2^-22: relative for 2^x, absolute for log2 x, whose argument here is a
// product of eight factors in [1, 2]).
__device__ inline float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ inline float lg2f(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kTopThreads, 1)
    router_top_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmhi,
                      const __grid_constant__ CUtensorMap tmlo, PrefillArgs a, Layout lay, float* __restrict__ dense,
                      int nblk_bh, unsigned long long* faults) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t afull[2], aempty[2], cfull[kTopStages], cempty[kTopStages], accfull[2], accempty[2];
  __shared__ int64_t off[kMaxLevels + 2];
  __shared__ LevelTab T;
  __shared__ int4 brec[2];  // per query-tile buffer: chunk count, pass-0 chunks, and N of chunks 2, 3 (8 bits each)
  __shared__ uint32_t tmem_base_sh;
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* abuf = smem;                       // [2][kTopABytes]
  unsigned char* cbuf = smem + 2 * kTopABytes;      // [kTopStages][kTopChunkBytes]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  load_offsets(lay, off);
  if (threadIdx.x == 0) {
    T.L = num_levels(a.N, a.C);
    T.lc = ilog2_pow2(a.C);
    for (int l = 1; l <= T.L; ++l) T.size[l] = level_size(a.N, a.C, l);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&afull[i], 1);
      mbar_init(&aempty[i], 1);
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 8);  // the eight warps of the pass's two epilogue groups
    }
    for (int i = 0; i < kTopStages; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cempty[i], 1);
    }
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kTopCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int nblk = a.B * a.H_kv * nblk_bh;
  auto block_pos = [&](int blk, int& bh, int64_t& i0, int64_t& t_last) {
    bh = blk / nblk_bh;
    i0 = static_cast<int64_t>(blk % nblk_bh) * kDenseQ;
    t_last = a.q0 + min(static_cast<int64_t>(a.Nq) - 1, i0 + kDenseQ - 1);
  };

  if (warp == kTopEpiWarps) {
    // ------------------------------------------------------ copies
    if (lane == 0) {
      int k = 0, n = 0;  // live blocks and chunks so far
      for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
        int bh;
        int64_t i0, t_last;
        block_pos(blk, bh, i0, t_last);
        const TopGeom g = top_geom(T, a.K, t_last, a.causal != 0);
        if (g.nl == 0) continue;
        const int ab = k & 1;
        mbar_wait(&aempty[ab], ((k >> 1) & 1) ^ 1, faults);
        const int b = bh / a.H_kv, h = bh % a.H_kv;
        const int nj = n_chunks_total(g);
        // The block's chunk schedule for the MMA thread, published by the
        // arrival below (the MMA thread reads it after waiting on afull).
        brec[ab] = make_int4(nj, g.nl < 2 ? g.nl : 2, chunk_rows(g, 0) | (nj > 1 ? chunk_rows(g, 1) << 8 : 0),
                             (nj > 2 ? chunk_rows(g, 2) : 0) | (nj > 3 ? chunk_rows(g, 3) << 8 : 0));
        mbar_expect_tx(&afull[ab], kTopABytes);
        tma_load_3d(abuf + ab * kTopABytes, &tmq, 0, b * a.H_q + 8 * h, static_cast<int>(i0), &afull[ab]);
        tma_load_3d(abuf + ab * kTopABytes + kTopABytes / 2, &tmq, 64, b * a.H_q + 8 * h, static_cast<int>(i0),
                    &afull[ab]);
        const int64_t row_base = static_cast<int64_t>(bh) * lay.R;
        for (int j = 0; j < nj; ++j, ++n) {
          const int i = chunk_level(j);
          const int y = static_cast<int>(row_base + off[g.lev[i] - 1] + (j < 2 ? 0 : kTopChunkRows * (j - 2)));
          const int s = n % kTopStages;
          mbar_wait(&cempty[s], ((n / kTopStages) & 1) ^ 1, faults);
          unsigned char* dst = cbuf + s * kTopChunkBytes;
          mbar_expect_tx(&cfull[s], kTopChunkBytes);
          tma_load_2d(dst, &tmhi, 0, y, &cfull[s]);
          tma_load_2d(dst + kTopHalf, &tmhi, 64, y, &cfull[s]);
          tma_load_2d(dst + 2 * kTopHalf, &tmlo, 0, y, &cfull[s]);
          tma_load_2d(dst + 3 * kTopHalf, &tmlo, 64, y, &cfull[s]);
        }
        ++k;
      }
      // End record: the MMA thread stops at a block without chunks.
      const int ab = k & 1;
      mbar_wait(&aempty[ab], ((k >> 1) & 1) ^ 1, faults);
      brec[ab] = make_int4(0, 0, 0, 0);
      mbar_arrive(&afull[ab]);
    }
  } else if (warp == kTopEpiWarps + 1) {
    // ------------------------------------------------------ MMAs
    if (lane == 0) {
      // Operand descriptors differ from the buffer's base descriptor only in
      // the start-address field (16-byte units, no carry below 256 KB).
      const uint64_t da = sw128_desc(smem_u32(abuf)), dc = sw128_desc(smem_u32(cbuf));
      int n = 0, npass0 = 0, npass1 = 0;
      for (int k = 0;; ++k) {  // the copy thread's blocks, until its end record (no chunks)
        const int ab = k & 1;
        if (!mbar_wait(&afull[ab], (k >> 1) & 1, faults)) break;
        const int4 rec = brec[ab];
        const int nj = rec.x, n0 = rec.y;
        if (nj == 0) break;
        const uint64_t dab = da + ((ab * kTopABytes) >> 4);
        for (int j = 0; j < nj; ++j, ++n) {
          if (j == 0) mbar_wait(&accempty[0], (npass0 & 1) ^ 1, faults);  // pass 0's groups are done with it
          if (j == 2) mbar_wait(&accempty[1], (npass1 & 1) ^ 1, faults);
          const int s = n % kTopStages;
          mbar_wait(&cfull[s], (n / kTopStages) & 1, faults);
          tc_fence_after();
          const uint64_t dcs = dc + ((s * kTopChunkBytes) >> 4);
          const uint32_t dcol = tmem + chunk_col(j);
          const int rows = ((j < 2 ? rec.z : rec.w) >> (8 * (j & 1))) & 0xff;
          const uint32_t idesc = idesc_n(rows);  // only the chunk's rows that hold children
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint32_t ao = (ks >> 2) * (kTopABytes / 2) + (ks & 3) * 32;
              const uint32_t bo = part * 2 * kTopHalf + (ks >> 2) * kTopHalf + (ks & 3) * 32;
              umma_bf16(dcol, dab + (ao >> 4), dcs + (bo >> 4), idesc, (part | ks) != 0);
            }
          }
          umma_commit(&cempty[s]);
          if (j + 1 == n0) {
            umma_commit(&accfull[0]);
            ++npass0;
          } else if (j >= 2 && j + 1 == nj) {
            umma_commit(&accfull[1]);
            ++npass1;
          }
        }
        umma_commit(&aempty[ab]);
      }
    }
  } else {
    // ------------------------------------------------------ epilogue
    const int grp = warp >> 2, qtr = warp & 3;   // group: 0 level 0, 1 level 1, 2 / 3 level 2 halves
    const int p = grp < 2 ? 0 : 1;               // the pass (TMEM accumulator) it reads
    const int r = 32 * qtr + lane;               // TMEM lane = tile row
    const int qi = r >> 3, hd = r & 7;           // query of the block, head of the group
    const bool causal = a.causal != 0;
    int npass = 0;
    for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
      int bh;
      int64_t i0, t_last;
      block_pos(blk, bh, i0, t_last);
      const TopGeom g = top_geom(T, a.K, t_last, a.causal != 0);
      if (g.nl == 0 || (p == 1 && g.nl < 3)) continue;  // the pass does not exist for this block
      mbar_wait(&accfull[p], npass & 1, faults);
      __syncwarp();
      tc_fence_after();
      const int i = grp < 2 ? grp : 2;
      if (i < g.nl) {
        const int64_t i_row = i0 + qi;
        const bool live = i_row < a.Nq;
        const int64_t t = a.q0 + (live ? i_row : a.Nq - 1);
        float* drow = dense + (static_cast<int64_t>(bh) * a.Nq + (live ? i_row : 0)) * kDenseSlots + dense_slot0(i);
        const int l = g.lev[i];
        const int vcl = static_cast<int>(tab_valid(T, l, t, causal));
        const int vcc = static_cast<int>(tab_valid(T, l - 1, t, causal));
        const int c_lo = grp == 3 ? 64 : 0, c_hi = grp == 2 ? min(g.nn[i], 64) : g.nn[i];
        const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * qtr) << 16) + chunk_col(i < 2 ? i : 2);
        // 16 nodes per 32-column load; the node range is the same for the
        // whole group, so its four warps run the same loop.
        for (int c0 = c_lo; c0 < c_hi; c0 += 16) {
          uint32_t v[32];
          tmem_ld32(tbase + 2 * c0, v);
          tmem_ld_wait();
          // Per head, log(e^s0 + e^s1) = max + log(1 + e^-|s0 - s1|); over the
          // 8 heads the maxima add and the (1 + e^-|d|) factors multiply, so
          // one exponential per (node, head) and one logarithm per node.
          float mx[16], pr[16];
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const float s0 = a.scale * __uint_as_float(v[2 * m]), s1 = a.scale * __uint_as_float(v[2 * m + 1]);
            const bool two = 2 * (c0 + m) + 1 < vcc;
            mx[m] = two ? fmaxf(s0, s1) : s0;
            pr[m] = two ? 1.f + ex2f(-fabsf(s0 - s1) * 1.4426950408889634f) : 1.f;
          }
          // Sum of the maxima and product of the factors over the 8 heads
          // (lanes 8 j .. 8 j + 7) by a reduce-scatter: each step keeps one
          // half of the nodes and combines the partner's values of that half;
          // afterwards lane hd holds nodes c0 + 2 hd and c0 + 2 hd + 1.
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const bool up = hd & 4;
            const float sm = up ? mx[k] : mx[k + 8], km = up ? mx[k + 8] : mx[k];
            const float sp = up ? pr[k] : pr[k + 8], kp = up ? pr[k + 8] : pr[k];
            mx[k] = km + __shfl_xor_sync(kFull, sm, 4);
            pr[k] = kp * __shfl_xor_sync(kFull, sp, 4);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const bool up = hd & 2;
            const float sm = up ? mx[k] : mx[k + 4], km = up ? mx[k + 4] : mx[k];
            const float sp = up ? pr[k] : pr[k + 4], kp = up ? pr[k + 4] : pr[k];
            mx[k] = km + __shfl_xor_sync(kFull, sm, 2);
            pr[k] = kp * __shfl_xor_sync(kFull, sp, 2);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const bool up = hd & 1;
            const float sm = up ? mx[k] : mx[k + 2], km = up ? mx[k + 2] : mx[k];
            const float sp = up ? pr[k] : pr[k + 2], kp = up ? pr[k + 2] : pr[k];
            mx[k] = km + __shfl_xor_sync(kFull, sm, 1);
            pr[k] = kp * __shfl_xor_sync(kFull, sp, 1);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int c = c0 + 2 * hd + k;
            if (live && c < vcl) drow[c] = mx[k] + lg2f(pr[k]) * 0.6931471805599453f;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[p]);
      ++npass;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTopCols);
  }
}

}  // namespace

// The shapes its parity tests cover (the tcgen05 leaf scorer's: C = 64).
bool router_top_supported(const PrefillArgs& a) {
  return a.dtype == PISA_DTYPE_BF16 && a.d == 128 && a.H_q == 8 * a.H_kv && a.K <= 16 && a.C == 64;
}

cudaError_t launch_router_top(const PrefillArgs& a, const void* q, const Layout& lay, const Ws& ws, cudaStream_t st) {
  // Queries as (d, head, position): a box of 64 columns x 8 heads x 16
  // positions lands as 128 rows (query, head) of 128 bytes.
  CUtensorMap tmq, tmhi, tmlo;
  cudaError_t e = make_tmap_bf16_3d_strided(&tmq, q, 128, static_cast<uint64_t>(a.B) * a.H_q,
                                            static_cast<uint64_t>(a.Nq), static_cast<uint64_t>(a.Nq) * 256, 256, 8,
                                            kDenseQ);
  const uint64_t prow = static_cast<uint64_t>(a.B) * a.H_kv * lay.R;
  if (e == cudaSuccess) e = make_tmap_bf16_2d(&tmhi, ws.hi, 128, prow, kTopChunkRows);
  if (e == cudaSuccess) e = make_tmap_bf16_2d(&tmlo, ws.lo, 128, prow, kTopChunkRows);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(router_top_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTopSmem);
  if (e != cudaSuccess) return e;
  const int nblk_bh = static_cast<int>((static_cast<int64_t>(a.Nq) + kDenseQ - 1) / kDenseQ);
  const int64_t nblk = static_cast<int64_t>(a.B) * a.H_kv * nblk_bh;
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  const int grid = static_cast<int>(nblk < sms ? nblk : sms);
  if (grid <= 0) return cudaSuccess;
  TimedLaunch tl("router_top_kernel", st);
  router_top_kernel<<<grid, kTopThreads, kTopSmem, st>>>(tmq, tmhi, tmlo, a, lay, ws.dense, nblk_bh,
                                                         wait_fault_counter());
  count_launch();
  return cudaGetLastError();
}

}  // namespace pisa
