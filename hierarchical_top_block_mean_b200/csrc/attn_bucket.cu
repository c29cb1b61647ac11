// Block-sparse attention forward by leaf bucket, for bf16 prefill with
// d = 128, C = 64 and G_Q in {4, 8} (paper §BSA):
//   o_t = sum_{j in T_t} exp(scale q_t.k_j) v_j / sum_{j in T_t} exp(scale q_t.k_j).
//
// The selection is inverted, as stage 2 of the selection does for its
// candidates: the (query row, slot) pairs of each (kv head, query window,
// leaf) bucket form a list, cut into work items of kAbItemPairs pairs. Each
// item loads its leaf's K tile and V^T tile once and passes its queries by in
// tiles of 128 (query, head) rows, so a K/V tile serves every query of the
// window that selected it instead of being gathered once per query. Per tile
// (tcgen05, accumulators in TMEM):
//   S [128 rows x 64 keys]  = Q K^T                  (Q gathered by cp.async)
//   P = exp(scale S - m) per row over its usable keys, m the row maximum,
//       l = sum of P (bf16 P written to shared memory as the next A operand)
//   O [128 rows x 128 d]    = P V                    (B = V^T, K-major)
// and each pair writes its partial (m, l, O) per head, O unnormalised; l sums
// the fp32 P (the O MMA takes P rounded to bf16). attn_merge_kernel then
// combines the K partials of every (query, head) in slot order:
//   M = max m_k, L = sum l_k e^{m_k - M}, o = sum (e^{m_k - M} / L) O_k,
//   lse = M + log L.
// The result of a pair does not depend on which other pairs share its tile,
// and the merge order is fixed, so the output is reproducible bit for bit.
//
// Kernels: attn_vt_kernel (V^T into the workspace), attn_count_kernel,
// attn_scan_kernel, attn_scatter_kernel, attn_itemize_kernel (the inversion),
// attn_bucket_kernel (partials), attn_merge_kernel.
//
// attn_bucket_kernel is persistent (one CTA per SM) and warp-specialised:
//   warps 16-17 (loads): per tile, the 128 (query, head) rows by 16-byte
//     cp.async into a ring of kAbQStages 128-byte-swizzled stages;
//   warp 18, one lane: per item the K and V^T tiles by bulk tensor copy
//     (double buffered, requested as soon as a stage frees); it polls the
//     pipeline, issuing each tile's S MMAs and, once the tile's P is in
//     shared memory, its O MMAs, whichever is ready first;
//   warps 0-15 (epilogue): four groups of four warps take tiles in turn
//     (group = TMEM stage = tile index mod 4); each thread owns one (query,
//     head) row. A stage's S columns are overwritten by its O once the group
//     has formed P, and the stage takes a new tile once O has been read.
// Every mbarrier wait is bounded in time; the TMEM allocation is released
// before exit.
#include <algorithm>

#include "dispatch.cuh"
#include "kernels.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace pisa {

namespace {

constexpr int kAbItemPairs = 128;  // pairs per work item (64 measured 2 % slower at 256K)
constexpr int kAbGroups = 4;                    // epilogue groups = TMEM stages
constexpr int kAbEpiWarps = 4 * kAbGroups;
constexpr int kAbLoadWarps = 2;
constexpr int kAbMmaWarp = kAbEpiWarps + kAbLoadWarps;
constexpr int kAbThreads = 32 * (kAbMmaWarp + 1);
constexpr int kAbLoaders = 32 * kAbLoadWarps;
constexpr int kAbQStages = 3;
constexpr int kAbQBytes = 128 * 128 * 2;        // 128 rows x 128 bf16 (two 64-column halves)
constexpr int kAbKBytes = 64 * 128 * 2;         // 64 keys x 128 d (two halves)
constexpr int kAbVBytes = 128 * 64 * 2;         // 128 d x 64 keys (one box)
constexpr int kAbPBytes = 128 * 64 * 2;         // 128 rows x 64 keys
constexpr int kAbSmem = 1024 + 2 * (kAbKBytes + kAbVBytes) + kAbQStages * kAbQBytes + kAbGroups * kAbPBytes;
// Stage s occupies TMEM columns [128 s, 128 s + 128): S in its first 64, then
// O over all 128 once S has been read.
constexpr uint32_t kAbTmemCols = 512;
// Instruction descriptors (kind::f16, bf16 A and B, fp32 D, both K-major).
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescO = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct AbWs {
  int32_t* count;       // [nb] pairs per bucket
  int32_t* rank;        // [rows K] each selected (row, slot) entry's position in its bucket
  int32_t* off;         // [nb + 1] bucket offsets
  int32_t* item_off;    // [nb + 1] item offsets
  uint32_t* pairs;      // [rows K] (query row << 5 | slot), grouped by bucket
  int4* item_info;      // [items] {bh, first pair, end pair, leaf}
  bf16* vt;             // [B H_kv][128][Np] V transposed, keys padded to Np
  bf16* part_o;         // [rows K][16 chunks][G][8] O_k (unnormalised) per (pair, head)
  float2* part_ml;      // [rows K G] (m_k, l_k)
  int win_shift, nwin;
  int64_t Np;
};

inline size_t ab_al(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Query window of the (kv head, window, block) buckets: about 256 MB of one
// kv head's queries. Measured at 256K, G_Q = 8: windows of 8 / 16 / 32 / 64 /
// 128 / 256 / 512 MB gave 8.24 / 7.11 / 6.58 / 6.39 / 6.28 / 6.17 / 6.15 ms
// for the partials kernel. Fewer buckets mean fewer K and V tile loads and
// fuller tiles, and that outweighs keeping the window's queries in L2.
inline int ab_window_shift(const PrefillArgs& a) {
  const int64_t per_query = static_cast<int64_t>(a.H_q / a.H_kv) * a.d * 2;
  int sh = 6;
  while ((int64_t{1} << (sh + 1)) * per_query <= (int64_t{256} << 20) && sh < 30) ++sh;
  return sh;
}

size_t ab_carve(const PrefillArgs& a, char* base, AbWs* w) {
  const int G = a.H_q / a.H_kv;
  const size_t rows = static_cast<size_t>(a.B) * a.H_kv * a.Nq;
  const int sh = ab_window_shift(a);
  const int nwin = static_cast<int>((static_cast<int64_t>(a.Nq) + (int64_t{1} << sh) - 1) >> sh);
  const int64_t M1 = level_size(a.N, a.C, 1);
  const size_t nb = static_cast<size_t>(a.B) * a.H_kv * nwin * M1;
  const int64_t Np = (static_cast<int64_t>(a.N) + 63) / 64 * 64;
  const size_t items = rows * a.K / kAbItemPairs + nb + 1;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + o : nullptr;
    o += ab_al(bytes);
    return p;
  };
  AbWs x;
  x.count = reinterpret_cast<int32_t*>(take(nb * 4));
  x.rank = reinterpret_cast<int32_t*>(take(rows * a.K * 4));
  x.off = reinterpret_cast<int32_t*>(take((nb + 1) * 4));
  x.item_off = reinterpret_cast<int32_t*>(take((nb + 1) * 4));
  x.pairs = reinterpret_cast<uint32_t*>(take(rows * a.K * 4));
  x.item_info = reinterpret_cast<int4*>(take(items * 16));
  x.vt = reinterpret_cast<bf16*>(take(static_cast<size_t>(a.B) * a.H_kv * 128 * Np * 2));
  x.part_o = reinterpret_cast<bf16*>(take(rows * a.K * G * 128 * 2));
  x.part_ml = reinterpret_cast<float2*>(take(rows * a.K * G * 8));
  x.win_shift = sh;
  x.nwin = nwin;
  x.Np = Np;
  if (w) *w = x;
  return o;
}

// ------------------------------------------------------------ V transpose
// V [bh][N][128] -> V^T [bh][128][Np] through 64 x 64 shared tiles; keys past
// N are written as zeros.
__global__ void __launch_bounds__(256) attn_vt_kernel(const bf16* __restrict__ v, bf16* __restrict__ vt, int64_t N,
                                                      int64_t Np) {
  __shared__ bf16 tile[64][66];
  const int64_t bh = blockIdx.z;
  const int64_t key0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int d0 = blockIdx.y * 64;
  const bf16* src = v + bh * N * 128;
  for (int i = threadIdx.x; i < 64 * 64; i += blockDim.x) {
    const int r = i >> 6, c = i & 63;  // r: key, c: d
    const int64_t key = key0 + r;
    tile[r][c] = key < N ? src[key * 128 + d0 + c] : __float2bfloat16_rn(0.f);
  }
  __syncthreads();
  bf16* dst = vt + bh * 128 * Np;
  for (int i = threadIdx.x; i < 64 * 64; i += blockDim.x) {
    const int r = i >> 6, c = i & 63;  // r: d, c: key
    dst[static_cast<int64_t>(d0 + r) * Np + key0 + c] = tile[c][r];
  }
}

// ------------------------------------------------------------ inversion
__device__ inline int64_t ab_bucket(const AbWs& w, int64_t bh, int64_t i_row, int64_t M1, int leaf) {
  return (bh * w.nwin + (i_row >> w.win_shift)) * M1 + leaf;
}

__global__ void __launch_bounds__(256) attn_count_kernel(const int32_t* __restrict__ sel, int64_t entries, int K,
                                                         int Nq, int64_t M1, AbWs w) {
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < entries;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int leaf = sel[x];
    if (leaf < 0 || leaf >= M1) continue;
    const int64_t row = x / K;
    w.rank[x] = atomicAdd(&w.count[ab_bucket(w, row / Nq, row % Nq, M1, leaf)], 1);  // place in the bucket
  }
}

// One CTA: exclusive scans of the bucket sizes and of the items per bucket.
__global__ void __launch_bounds__(1024) attn_scan_kernel(AbWs w, int nb) {
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
      c[j] = i < nb ? w.count[i] : 0;
      it[j] = (c[j] + kAbItemPairs - 1) / kAbItemPairs;
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
        w.off[i] = e0;
        w.item_off[i] = e1;
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
    w.off[nb] = carry[0];
    w.item_off[nb] = carry[1];
  }
}

__global__ void __launch_bounds__(256) attn_scatter_kernel(const int32_t* __restrict__ sel, int64_t entries, int K,
                                                           int Nq, int64_t M1, AbWs w) {
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < entries;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int leaf = sel[x];
    if (leaf < 0 || leaf >= M1) continue;
    const int64_t row = x / K;
    const int slot = static_cast<int>(x % K);
    const int64_t i_row = row % Nq;
    const int64_t b = ab_bucket(w, row / Nq, i_row, M1, leaf);
    const int pos = w.rank[x];
    w.pairs[w.off[b] + pos] = (static_cast<uint32_t>(i_row) << 5) | static_cast<uint32_t>(slot);
  }
}

__global__ void __launch_bounds__(256) attn_itemize_kernel(AbWs w, int nb, int64_t M1) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nb) return;
  const int i0 = w.item_off[b], i1 = w.item_off[b + 1];
  const int p0 = w.off[b], p1 = w.off[b + 1];
  const int bh = static_cast<int>(b / (w.nwin * M1));
  const int leaf = static_cast<int>(b % M1);
  for (int i = i0; i < i1; ++i) {
    const int lo = p0 + (i - i0) * kAbItemPairs;
    w.item_info[i] = make_int4(bh, lo, min(lo + kAbItemPairs, p1), leaf);
  }
}

// ------------------------------------------------------------ partials
template <int G>
__global__ void __launch_bounds__(kAbThreads, 1)
    attn_bucket_kernel(const bf16* __restrict__ q, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmvt, PrefillArgs a, AbWs ws, int nb,
                       unsigned long long* faults) {
  constexpr int TQ = 128 / G;  // queries per tile
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t kvfull[2], kvempty[2], qfull[kAbQStages], qempty[kAbQStages];
  __shared__ uint64_t sfull[kAbGroups], pfull[kAbGroups], ofull[kAbGroups], tfree[kAbGroups];
  __shared__ uint32_t tmem_base_sh;
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* kbuf = smem;                                   // [2][kAbKBytes]
  unsigned char* vbuf = kbuf + 2 * kAbKBytes;                   // [2][kAbVBytes]
  unsigned char* qbuf = vbuf + 2 * kAbVBytes;                   // [kAbQStages][kAbQBytes]
  unsigned char* pbuf = qbuf + kAbQStages * kAbQBytes;          // [kAbGroups][kAbPBytes]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kvfull[i], 1);
      mbar_init(&kvempty[i], 1);
    }
    for (int i = 0; i < kAbGroups; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 4);
      mbar_init(&ofull[i], 1);
      mbar_init(&tfree[i], 4);
    }
    for (int i = 0; i < kAbQStages; ++i) {
      mbar_init(&qfull[i], kAbLoaders);
      mbar_init(&qempty[i], 1);
    }
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kAbTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  const int total = ws.item_off[nb];
  const bool causal = a.causal != 0;
  auto info = [&](int item) { return item < total ? ws.item_info[item] : make_int4(0, 0, 0, 0); };
  // Tile stream of this CTA: items blockIdx.x, + gridDim.x, ..., each cut
  // into tiles of TQ pairs.
  struct Stream {
    int item, tl, ntiles;
    int4 inf, inf_next;
  };
  auto ntiles_of = [&](int4 inf) { return (inf.z - inf.y + TQ - 1) / TQ; };
  auto stream_begin = [&]() {
    Stream st;
    st.item = blockIdx.x;
    st.tl = 0;
    st.inf = info(st.item);
    st.ntiles = ntiles_of(st.inf);
    st.inf_next = info(st.item + gridDim.x);
    return st;
  };
  auto stream_next = [&](Stream st) {
    if (st.item < total && ++st.tl >= st.ntiles) {
      st.item += gridDim.x;
      st.tl = 0;
      if (st.item < total) {
        st.inf = st.inf_next;
        st.ntiles = ntiles_of(st.inf);
        st.inf_next = info(st.item + gridDim.x);
      }
    }
    return st;
  };

  if (warp >= kAbEpiWarps && warp < kAbMmaWarp) {
    // ---------------------------------------------------------- query loads
    // Thread (warp lw, lane l) copies 16-byte column jcol = l & 15 of rows
    // r = slot + 8 m (m = 0 .. 15) of each tile, slot = 2 lw + (l >> 4): row
    // r is head r % G of the tile's query r / G.
    const int lw = warp - kAbEpiWarps;
    const int jcol = lane & 15;
    const int64_t head_stride = static_cast<int64_t>(a.Nq) * 128;
    int nq = 0;
    auto tile_words = [&](const Stream& st) -> uint32_t {
      if (st.item >= total) return 0u;
      const int p0 = st.inf.y + st.tl * TQ;
      return lane < min(TQ, st.inf.z - p0) ? ws.pairs[p0 + lane] : 0xffffffffu;
    };
    Stream sm = stream_begin();
    uint32_t tw_next = tile_words(sm);
    while (sm.item < total) {
      const Stream cur = sm;
      const uint32_t twv = tw_next;
      sm = stream_next(sm);
      tw_next = tile_words(sm);
      const int64_t bh = cur.inf.x;
      const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
      const bf16* qg = q + (b * a.H_q + h * G) * head_stride + jcol * 8;  // head 0 of the group, this column
      const int qs = nq % kAbQStages;
      mbar_wait(&qempty[qs], ((nq / kAbQStages) & 1) ^ 1, faults);
      const uint32_t qd = smem_u32(qbuf + qs * kAbQBytes) + (jcol >> 3) * (kAbQBytes / 2);
#pragma unroll
      for (int sl = 0; sl < 8 / (2 * kAbLoadWarps); ++sl)
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int slot = 2 * lw + (lane >> 4) + 2 * kAbLoadWarps * sl;
        const int r = slot + 8 * m;
        const int qi = r / G, hd = r % G;
        const uint32_t wq = __shfl_sync(kFull, twv, qi);
        const uint32_t dst = qd + r * 128 + (((jcol & 7) ^ (r & 7)) << 4);
        // rows of absent queries are zero-filled by the copy itself
        const bool has = wq != 0xffffffffu;
        cp16_zfill(dst, has ? qg + hd * head_stride + static_cast<int64_t>(wq >> 5) * 128 : qg, has ? 16 : 0);
      }
      // The stage's barrier completes once every loader thread's copies so
      // far have landed; the MMA thread fences the async proxy after
      // observing it.
      cp_arrive_noinc(&qfull[qs]);
      ++nq;
    }
    cp_wait<0>();
  } else if (warp == kAbMmaWarp) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      // Item j of this CTA (item blockIdx.x + j gridDim.x) uses K/V stage
      // j & 1; the O MMAs of an item's last tile free it, and the tiles of
      // item j + 2 are requested at once. One thread issues every MMA, so it
      // never blocks on one epilogue group while the other could use the
      // tensor cores: it polls, issuing the oldest pending O MMAs once their
      // P is ready, and the next tile's S MMAs once its queries, its TMEM
      // stage and its K/V tile are (a new item first needs the O MMAs of the
      // item two back, its stage's last user). S runs in tile order and O in
      // tile order. With no progress for kWaitNs the loop gives up (counted
      // as a fault), like every bounded wait.
      // A K/V request waits in kv_pend[stage] (item j, its record loaded
      // when the request is made) until the stage's previous O MMAs have
      // completed; the polling loop issues it then, without blocking.
      // (Two named registers per stage rather than arrays, so that the
      // record's load is not waited for until the request is issued.)
      int kv_pend0 = -1, kv_pend1 = -1;
      int4 kv_inf0 = make_int4(0, 0, 0, 0), kv_inf1 = make_int4(0, 0, 0, 0);
      auto request_kv = [&](int j) {
        const int it = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
        if (it >= total) return;
        if (j & 1) {
          kv_pend1 = j;
          kv_inf1 = ws.item_info[it];
        } else {
          kv_pend0 = j;
          kv_inf0 = ws.item_info[it];
        }
      };
      auto try_issue_kv = [&](int kb) -> bool {
        const int j = kb ? kv_pend1 : kv_pend0;
        if (j < 0 || !mbar_test(&kvempty[kb], ((j >> 1) & 1) ^ 1)) return false;
        const int4 inf = kb ? kv_inf1 : kv_inf0;
        const int ky = static_cast<int>(static_cast<int64_t>(inf.x) * a.N + static_cast<int64_t>(inf.w) * 64);
        mbar_expect_tx(&kvfull[kb], kAbKBytes + kAbVBytes);
        tma_load_2d(kbuf + kb * kAbKBytes, &tmk, 0, ky, &kvfull[kb]);
        tma_load_2d(kbuf + kb * kAbKBytes + kAbKBytes / 2, &tmk, 64, ky, &kvfull[kb]);
        tma_load_2d(vbuf + kb * kAbVBytes, &tmvt, inf.w * 64, inf.x * 128, &kvfull[kb]);
        (kb ? kv_pend1 : kv_pend0) = -1;
        return true;
      };
      struct Pend {
        int n, j;
        bool last;
      };
      constexpr int kF = kAbGroups;  // S issued, O pending: at most one tile per TMEM stage
      Pend fifo[kF];
      int f_head = 0, f_len = 0;
      request_kv(0);
      request_kv(1);
      try_issue_kv(0);
      try_issue_kv(1);
      Stream sm = stream_begin();
      int n = 0, j = -1;
      uint64_t t_prog = global_ns();
      while (sm.item < total || f_len > 0) {
        bool prog = false;
        if (f_len > 0) {
          const Pend pd = fifo[f_head];
          const int s = pd.n % kAbGroups, u = pd.n / kAbGroups, kb = pd.j & 1;
          if (mbar_test(&pfull[s], u & 1)) {
            tc_fence_after();
            const uint32_t pa = smem_u32(pbuf + s * kAbPBytes), vb = smem_u32(vbuf + kb * kAbVBytes);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              umma_bf16(tmem + 128 * s, sw128_desc(pa + ks * 32), sw128_desc(vb + ks * 32), kIdescO, ks > 0);
            umma_commit(&ofull[s]);
            f_head = (f_head + 1) % kF;
            --f_len;
            if (pd.last) {
              umma_commit(&kvempty[kb]);
              request_kv(pd.j + 2);
            }
            prog = true;
          }
        }
        if (try_issue_kv(0)) prog = true;
        if (try_issue_kv(1)) prog = true;
        if (sm.item < total && f_len < kF) {
          const bool first = sm.tl == 0;
          const int jn = first ? j + 1 : j;
          const int s = n % kAbGroups, u = n / kAbGroups, qs = n % kAbQStages;
          bool ready = !(first && f_len > 0 && fifo[f_head].j <= jn - 2);
          ready = ready && (!first || mbar_test(&kvfull[jn & 1], (jn >> 1) & 1));
          ready = ready && mbar_test(&qfull[qs], (n / kAbQStages) & 1);
          ready = ready && mbar_test(&tfree[s], (u & 1) ^ 1);  // the group has read O of tile n - kAbGroups
          if (ready) {
            j = jn;
            fence_proxy_async();  // the loaders' cp.async writes, before the tensor cores read them
            tc_fence_after();
            const uint32_t qa = smem_u32(qbuf + qs * kAbQBytes), ka = smem_u32(kbuf + (j & 1) * kAbKBytes);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint32_t qo = (ks >> 2) * (kAbQBytes / 2) + (ks & 3) * 32;
              const uint32_t ko = (ks >> 2) * (kAbKBytes / 2) + (ks & 3) * 32;
              umma_bf16(tmem + 128 * s, sw128_desc(qa + qo), sw128_desc(ka + ko), kIdescS, ks > 0);
            }
            umma_commit(&qempty[qs]);
            umma_commit(&sfull[s]);
            fifo[(f_head + f_len) % kF] = Pend{n, j, sm.tl + 1 == sm.ntiles};
            ++f_len;
            sm = stream_next(sm);
            ++n;
            prog = true;
          }
        }
        if (prog) {
          t_prog = global_ns();
        } else if (global_ns() - t_prog > kWaitNs) {
          if (faults) atomicAdd(faults, 1ull);
          break;
        }
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const float sl2 = a.scale * 1.4426950408889634f;
    const int grp = warp >> 2, qtr = warp & 3;  // group grp takes tiles grp, grp + kAbGroups, ...
    const int r = 32 * qtr + lane;  // TMEM lane = tile row = query r / G, head r % G
    const int hd = r % G;
    auto row_word = [&](const Stream& st) -> uint32_t {
      if (st.item >= total) return 0xffffffffu;
      const int p = st.inf.y + st.tl * TQ + r / G;
      return p < st.inf.z ? ws.pairs[p] : 0xffffffffu;
    };
    auto advance = [&](Stream st) {
#pragma unroll
      for (int i = 0; i < kAbGroups; ++i) st = stream_next(st);
      return st;
    };
    Stream sm = stream_begin();
    int n = 0;
    for (; n < grp; ++n) sm = stream_next(sm);
    uint32_t w_next = row_word(sm);
    while (sm.item < total) {
      const int4 inf = sm.inf;
      const uint32_t w = w_next;
      const int ncur = n;
      sm = advance(sm);
      n += kAbGroups;
      w_next = row_word(sm);
      const int s = ncur % kAbGroups, u = ncur / kAbGroups;
      const bool ok = w != 0xffffffffu;
      const int64_t i_row = ok ? static_cast<int64_t>(w >> 5) : 0;
      const int64_t key0 = static_cast<int64_t>(inf.w) * 64;
      int nv = ok ? static_cast<int>(min(static_cast<int64_t>(64), a.N - key0)) : 0;
      if (causal && ok) nv = static_cast<int>(min(static_cast<int64_t>(nv), a.q0 + i_row - key0 + 1));
      mbar_wait(&sfull[s], u & 1, faults);
      __syncwarp();
      tc_fence_after();
      // S is read from TMEM twice, 32 columns at a time (maximum, then
      // exponentials), to keep the epilogue within the registers that four
      // groups of warps can hold.
      const uint32_t srow = tmem + (static_cast<uint32_t>(32 * qtr) << 16) + 128 * s;
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t v[32];
        tmem_ld32(srow + 32 * h2, v);
        tmem_ld_wait();
        if (nv >= 32 * h2 + 32) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) m4[jj & 3] = fmaxf(m4[jj & 3], __uint_as_float(v[jj]));
        } else {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (32 * h2 + jj < nv) m4[jj & 3] = fmaxf(m4[jj & 3], __uint_as_float(v[jj]));
        }
      }
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      const float mxs = nv > 0 ? mx * sl2 : 0.f;
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
      unsigned char* prow = pbuf + s * kAbPBytes + r * 128;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t v[32];
        tmem_ld32(srow + 32 * h2, v);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int jl = 8 * c + 2 * e, j0 = 32 * h2 + jl;
            const float p0 = j0 < nv ? ex2_approx(fmaf(__uint_as_float(v[jl]), sl2, -mxs)) : 0.f;
            const float p1 = j0 + 1 < nv ? ex2_approx(fmaf(__uint_as_float(v[jl + 1]), sl2, -mxs)) : 0.f;
            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            pk[e] = *reinterpret_cast<const uint32_t*>(&pb);
            l4[e] += p0 + p1;
          }
          const int cc = 4 * h2 + c;
          *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      const float l = (l4[0] + l4[1]) + (l4[2] + l4[3]);
      fence_proxy_async();  // the O MMA reads P through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(&pfull[s]);
      mbar_wait(&ofull[s], u & 1, faults);
      __syncwarp();
      tc_fence_after();
      // Partial layout per pair: [16 column chunks of 8][G heads][8] bf16, so
      // the G heads of a pair write each chunk as one contiguous piece. O is
      // stored unnormalised (P relative to the row maximum); (m, l) go beside it.
      const int64_t pair = (static_cast<int64_t>(inf.x) * a.Nq + i_row) * a.K + (ok ? (w & 31) : 0);
      bf16* dst = ws.part_o + pair * (G * 128) + hd * 8;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(srow + 32 * c, o);
        tmem_ld_wait();
        if (ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const __nv_bfloat162 ob = __floats2bfloat162_rn(__uint_as_float(o[e + 2 * f]), __uint_as_float(o[e + 2 * f + 1]));
              pk[f] = *reinterpret_cast<const uint32_t*>(&ob);
            }
            const int chunk = (32 * c + e) / 8;
            *reinterpret_cast<uint4*>(dst + chunk * (G * 8)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      if (ok) ws.part_ml[pair * G + hd] = make_float2(nv > 0 ? mx * a.scale : -INFINITY, l);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tfree[s]);  // the stage may take the next tile's S
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kAbTmemCols);
  }
}

// ------------------------------------------------------------ merge
// One warp per query row (b, kv head, t). Weights: lane L holds slot L & 15's
// (m, l) for heads 4 (L >> 4) .. 4 (L >> 4) + 3 (G = 8; G = 4 uses one head
// group), and the per-head max and sum over the slots are taken with
// shuffles. Outputs: lane L owns column chunk L >> 1 (8 columns) of heads
// hg = (L & 1) G / 2 .. + G / 2 - 1 and reads, per slot, the matching 16-byte
// pieces of the pair's partial block, so each slot's block is read whole
// and contiguously. Slots are combined in ascending order.
template <int G>
__global__ void __launch_bounds__(256) attn_merge_kernel(const int32_t* __restrict__ sel, PrefillArgs a, AbWs ws,
                                                         bf16* __restrict__ out, float* __restrict__ lse, int64_t rows) {
  constexpr int HG = G / 2;  // heads per lane in the output phase
  constexpr int HW = G / 2;  // heads per lane in the weight phase (two lane halves)
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int64_t bh = row / a.Nq, i_row = row % a.Nq;
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  const int K = a.K;
  const int64_t M1 = level_size(a.N, a.C, 1);
  const int selk = lane < K ? sel[row * K + lane] : -1;
  const unsigned valid = __ballot_sync(kFull, selk >= 0 && selk < M1);  // the slots that have a partial
  // ---- weights: lane (k = lane & 15, head group lane >> 4)
  const int wk = lane & 15, wg = lane >> 4;
  float m[HW], l[HW];
  const bool vk = (valid >> wk) & 1u;
#pragma unroll
  for (int i = 0; i < HW; ++i) {
    const float2 ml = vk ? ws.part_ml[(row * K + wk) * G + HW * wg + i] : make_float2(-INFINITY, 0.f);
    m[i] = ml.y > 0.f ? ml.x : -INFINITY;
    l[i] = ml.y > 0.f ? ml.y : 0.f;
  }
  float wt[HW], lse_h[HW];
#pragma unroll
  for (int i = 0; i < HW; ++i) {
    float M = m[i];
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    const float e = l[i] > 0.f ? expf(m[i] - M) : 0.f;  // scale of slot k's P relative to the row maximum
    float L = e * l[i];
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) L += __shfl_xor_sync(kFull, L, o);
    wt[i] = L > 0.f ? e / L : 0.f;
    lse_h[i] = M + logf(L);
  }
  // ---- outputs: lane (chunk lane >> 1, heads hg0 .. hg0 + HG - 1)
  const int chunk = lane >> 1, hg0 = (lane & 1) * HG;
  float acc[HG][8];
#pragma unroll
  for (int i = 0; i < HG; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
  const bf16* base = ws.part_o + (row * K) * (G * 128) + chunk * (G * 8) + hg0 * 8;
#pragma unroll 4
  for (int k = 0; k < 16; ++k) {
    if (k >= K || !((valid >> k) & 1u)) continue;  // warp-uniform
    uint4 x[HG];
#pragma unroll
    for (int i = 0; i < HG; ++i) x[i] = *reinterpret_cast<const uint4*>(base + static_cast<int64_t>(k) * (G * 128) + i * 8);
#pragma unroll
    for (int i = 0; i < HG; ++i) {
      // weight of (slot k, head hg0 + i): held by lane (k, head group (hg0 + i) / HW), entry (hg0 + i) % HW
      const int hh = hg0 + i;
      float wsel = 0.f;
#pragma unroll
      for (int j = 0; j < HW; ++j) {
        const float wj = __shfl_sync(kFull, wt[j], k + 16 * (hh / HW));
        if (j == hh % HW) wsel = wj;
      }
      const uint32_t u[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[i][2 * e] += wsel * __uint_as_float(u[e] << 16);
        acc[i][2 * e + 1] += wsel * __uint_as_float(u[e] & 0xffff0000u);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < HG; ++i) {
    const int hh = hg0 + i;
    const int64_t orow = (b * a.H_q + h * G + hh) * a.Nq + i_row;
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 ob = __floats2bfloat162_rn(acc[i][2 * e], acc[i][2 * e + 1]);
      pk[e] = *reinterpret_cast<const uint32_t*>(&ob);
    }
    *reinterpret_cast<uint4*>(out + orow * 128 + chunk * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  if (lse && wk == 0) {
#pragma unroll
    for (int i = 0; i < HW; ++i) lse[(b * a.H_q + h * G + HW * wg + i) * a.Nq + i_row] = lse_h[i];
  }
}

int ab_sm_count() {
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

bool attn_bucket_supported(const PrefillArgs& a) {
  const int G = a.H_q / a.H_kv;
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * a.Nq;
  return a.dtype == PISA_DTYPE_BF16 && a.d == 128 && a.C == 64 && (G == 4 || G == 8) && a.K <= 16 &&
         rows * a.K < (int64_t{1} << 31) && a.Nq < (1 << 27) &&
         static_cast<int64_t>(a.B) * a.H_kv * a.N + 64 < (int64_t{1} << 31) &&
         static_cast<int64_t>(a.B) * a.H_kv * 128 < (int64_t{1} << 31);
}

size_t attn_bucket_workspace_bytes(const PrefillArgs& a) {
  return attn_bucket_supported(a) ? ab_carve(a, nullptr, nullptr) : 0;
}

cudaError_t launch_attn_bucket(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                               void* out, float* lse, void* ws_ptr, cudaStream_t st) {
  AbWs w;
  ab_carve(a, static_cast<char*>(ws_ptr), &w);
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * a.Nq;
  const int64_t M1 = level_size(a.N, a.C, 1);
  const int nb = static_cast<int>(static_cast<int64_t>(a.B) * a.H_kv * w.nwin * M1);
  const int64_t entries = rows * a.K;
  cudaError_t e = cudaMemsetAsync(w.count, 0, static_cast<size_t>(nb) * 4, st);
  if (e != cudaSuccess) return e;
  const int sms = ab_sm_count();
  const unsigned eg = static_cast<unsigned>(std::min<int64_t>((entries + 255) / 256, static_cast<int64_t>(sms) * 32));
  {
    TimedLaunch tl("attn_vt_kernel", st);
    attn_vt_kernel<<<dim3(static_cast<unsigned>(w.Np / 64), 2, static_cast<unsigned>(a.B * a.H_kv)), 256, 0, st>>>(
        static_cast<const bf16*>(v), w.vt, a.N, w.Np);
  }
  count_launch();
  {
    TimedLaunch tl("attn_count_kernel", st);
    attn_count_kernel<<<eg, 256, 0, st>>>(sel, entries, a.K, a.Nq, M1, w);
  }
  count_launch();
  {
    TimedLaunch tl("attn_scan_kernel", st);
    attn_scan_kernel<<<1, 1024, 0, st>>>(w, nb);
  }
  count_launch();
  {
    TimedLaunch tl("attn_scatter_kernel", st);
    attn_scatter_kernel<<<eg, 256, 0, st>>>(sel, entries, a.K, a.Nq, M1, w);
  }
  count_launch();
  {
    TimedLaunch tl("attn_itemize_kernel", st);
    attn_itemize_kernel<<<static_cast<unsigned>((nb + 255) / 256), 256, 0, st>>>(w, nb, M1);
  }
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap tmk, tmvt;
  if ((e = make_tmap_bf16_2d(&tmk, k, 128, static_cast<uint64_t>(a.B) * a.H_kv * a.N, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&tmvt, w.vt, static_cast<uint64_t>(w.Np), static_cast<uint64_t>(a.B) * a.H_kv * 128,
                             128)) != cudaSuccess)
    return e;
  unsigned long long* faults = wait_fault_counter();
  return dispatch_tdg(PISA_DTYPE_BF16, 128, a.H_q / a.H_kv, [&](auto, auto, auto gg) -> cudaError_t {
    constexpr int G = decltype(gg)::value;
    if constexpr (G == 4 || G == 8) {
      auto kern = attn_bucket_kernel<G>;
      cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kAbSmem);
      if (e2 != cudaSuccess) return e2;
      {
        TimedLaunch tl("attn_bucket_kernel", st);
        kern<<<static_cast<unsigned>(sms), kAbThreads, kAbSmem, st>>>(static_cast<const bf16*>(q), tmk, tmvt, a, w, nb,
                                                                      faults);
      }
      count_launch();
      if ((e2 = cudaGetLastError()) != cudaSuccess) return e2;
      {
        TimedLaunch tl("attn_merge_kernel", st);
        attn_merge_kernel<G><<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(
            sel, a, w, static_cast<bf16*>(out), lse, rows);
      }
      count_launch();
      return cudaGetLastError();
    } else {
      return cudaErrorInvalidValue;
    }
  });
}

}  // namespace pisa
