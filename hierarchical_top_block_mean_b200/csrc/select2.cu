// Two-stage PISA selection for bf16 inputs (paper §Kernels, training and
// prefill kernels):
//   stage 1  router_top_kernel (router_top.cu; G_Q = 8, d = 128) every node
//                              of the top three scored levels of each block
//                              of 16 queries, on tcgen05;
//            router_kernel     one warp per (kv head, query): levels L..2 of
//                              the coarse-to-fine search, reading those node
//                              scores where present, else scoring the
//                              candidates' children on tensor cores.
//   grouping count (in stage 1), scan_kernel, scatter_kernel,
//                              itemize_kernel: a CSR of the (query, candidate
//                              leaf) pairs keyed by (kv head, query window,
//                              leaf), cut into work items of 128 pairs.
//   stage 2  leaf_umma_kernel  (leaf_umma.cu; G_Q = 8, d = 128, C = 64) or
//            leaf_kernel       per work item: the C x d key tile is brought
//                              into shared memory once and reused across
//                              tiles of the item's queries x G_Q heads
//                              ((Q_tile G_Q) x d . d x C on tensor cores),
//                              then a per-head LSE over the keys and a sum
//                              over the G_Q heads.
//   final    final_kernel      top K of each row's leaf scores.
//
// Numerics: queries and keys are bf16, so q.k products are exact in a bf16
// MMA with fp32 accumulation. Pyramid summaries are fp32; the router splits
// each into bf16 hi + lo and issues two MMAs, which reproduces the fp32
// summary to ~2^-16 relative.
#include "dispatch.cuh"
#include "mma.cuh"
#include "rowops.cuh"
#include "select2.cuh"
#include "select2_ws.cuh"
#include "tma.cuh"

namespace pisa {

namespace {

constexpr int kRouterWarps = 4;
constexpr int kPairsPerItem = 128;  // stage-2 work item (64 measured 6 % slower at 256K: more key-tile loads)
constexpr int kQTile = 4;
constexpr int kLeafThreads = 256;

// Query window of the stage-2 buckets: about 128 MB of one kv head's queries
// (W x G_Q x d x 2 bytes). All CTAs walk the buckets of one window at a time,
// so its query rows are read again while they are recent. Measured at 256K,
// G_Q = 8: windows of 16 / 32 / 64 / 128 / 1024 MB gave 6.0 / 5.85 / 5.60 /
// 5.48 / 5.47 ms of leaf scoring. A larger window has fewer (window, leaf)
// buckets, so fewer key-tile loads and ragged last tiles, and that outweighs
// the query rows that no longer stay in L2.
inline int window_shift(const PrefillArgs& a) {
  const int64_t per_query = static_cast<int64_t>(a.H_q / a.H_kv) * a.d * 2;
  int sh = 6;
  while ((int64_t{1} << (sh + 1)) * per_query <= (int64_t{128} << 20) && sh < 30) ++sh;
  return sh;
}

inline size_t al(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t carve(const PrefillArgs& a, char* base, Ws* w) {
  const size_t rows = static_cast<size_t>(a.B) * a.H_kv * a.Nq;
  const int sh = window_shift(a);
  const int nwin = static_cast<int>((static_cast<int64_t>(a.Nq) + (int64_t{1} << sh) - 1) >> sh);
  const size_t nb = static_cast<size_t>(a.B) * a.H_kv * nwin * level_size(a.N, a.C, 1);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + o : nullptr;
    o += al(bytes);
    return p;
  };
  Ws x;
  x.cand = reinterpret_cast<int32_t*>(take(rows * 32 * 4));
  x.ncand = reinterpret_cast<int32_t*>(take(rows * 4));
  x.score = reinterpret_cast<float*>(take(rows * 32 * 4));
  x.count = reinterpret_cast<int32_t*>(take(nb * 4));
  x.rank = reinterpret_cast<int32_t*>(take(rows * 32 * 4));
  x.bucket_off = reinterpret_cast<int32_t*>(take((nb + 1) * 4));
  x.item_off = reinterpret_cast<int32_t*>(take((nb + 1) * 4));
  x.pairs = reinterpret_cast<uint32_t*>(take(rows * 32 * 4));
  const size_t prow = static_cast<size_t>(a.B) * a.H_kv * make_layout(a.N, a.C).R;
  x.planes = reinterpret_cast<uint4*>(take(prow * a.d * 4));
  const bool top = router_top_supported(a);
  x.hi = top ? reinterpret_cast<bf16*>(take(prow * a.d * 2)) : nullptr;
  x.lo = top ? reinterpret_cast<bf16*>(take(prow * a.d * 2)) : nullptr;
  x.dense = top ? reinterpret_cast<float*>(take(rows * kDenseSlots * 4)) : nullptr;
  x.item_bucket = reinterpret_cast<int32_t*>(take((rows * 32 / kPairsPerItem + nb + 1) * 4));
  x.item_info = reinterpret_cast<int4*>(take((rows * 32 / kPairsPerItem + nb + 1) * 16));
  x.win_shift = sh;
  x.nwin = nwin;
  if (w) *w = x;
  return o;
}

// Pyramid rows (fp32) -> interleaved bf16 hi/lo chunks, so that the router
// reads ready MMA operands: chunk c of a row holds hi(x[4c..4c+3]) then
// lo(x[4c..4c+3]), with x - hi - lo below 2^-16 |x|.
__global__ void __launch_bounds__(256) split_kernel(const float4* __restrict__ pyr, uint4* __restrict__ planes,
                                                   uint2* __restrict__ hi, uint2* __restrict__ lo, int64_t n4) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 x = pyr[i];
    float h[4], l[4];
    split_bf16(x.x, h[0], l[0]);
    split_bf16(x.y, h[1], l[1]);
    split_bf16(x.z, h[2], l[2]);
    split_bf16(x.w, h[3], l[3]);
    const uint4 v = make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]), pack_bf16(l[0], l[1]), pack_bf16(l[2], l[3]));
    planes[i] = v;
    if (hi) {  // the same parts as plain row-major planes, for the tensor-memory router levels
      hi[i] = make_uint2(v.x, v.y);
      lo[i] = make_uint2(v.z, v.w);
    }
  }
}

// ---------------------------------------------------------------- stage 1
template <int D, int G>
__global__ void __launch_bounds__(kRouterWarps * 32)
    router_kernel(const bf16* __restrict__ q, const float* __restrict__ pyr, Layout lay, PrefillArgs a, Ws ws,
                  int32_t* __restrict__ sel, float* __restrict__ sel_score) {
  __shared__ int tmp[kRouterWarps][32];
  __shared__ int64_t off[kMaxLevels + 2];
  load_offsets(lay, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRouterWarps + warp;
  if (row >= static_cast<int64_t>(a.B) * a.H_kv * a.Nq) return;
  const int64_t n = a.N;
  const int64_t bh = row / a.Nq, i_row = row % a.Nq, t = a.q0 + i_row;  // query row and its position
  const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
  const bool causal = a.causal != 0;
  const int C = a.C, K = a.K;
  const uint4* PL = ws.planes + bh * lay.R * (D / 4);
  const float nanv = __int_as_float(0x7fffffff);

  int l = num_levels(n, C);
  while (l >= 1 && valid_count(n, C, l, t, causal) <= K) --l;
  if (l < 1) {  // the leaf level itself has <= K usable blocks: keep them all
    const int nv = static_cast<int>(valid_count(n, C, 1, t, causal));
    if (lane < K) {
      sel[row * K + lane] = lane < nv ? lane : -1;
      if (sel_score) sel_score[row * K + lane] = nanv;
    }
    if (lane == 0) ws.ncand[row] = -1;
    return;
  }
  int cand = lane < valid_count(n, C, l, t, causal) ? lane : -1;

  if (l >= 2) {
    // Query heads of the group as the B operand (columns = heads, zero padded to 8).
    uint32_t qb[D / 16][2];
    const int hd = gid < G ? gid : G - 1;
    const bf16* qrow = q + ((b * a.H_q + h * G + hd) * a.Nq + i_row) * D + 4 * tig;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint2 u = *reinterpret_cast<const uint2*>(qrow + 16 * ks);
      qb[ks][0] = gid < G ? u.x : 0u;
      qb[ks][1] = gid < G ? u.y : 0u;
    }
    // Levels whose node scores the tensor-memory pass has written: the top
    // three scored levels of this row's block of kDenseQ queries.
    int ltop = -1;
    const float* drow = nullptr;
    if (ws.dense) {
      const int64_t last = min(static_cast<int64_t>(a.Nq) - 1, (i_row / kDenseQ) * kDenseQ + kDenseQ - 1);
      ltop = start_level(n, C, K, a.q0 + last, causal);
      drow = ws.dense + row * kDenseSlots;
    }
    // Usable blocks of a level are exactly the first valid_count of them, so
    // one count per level replaces a per-candidate test.
    int vc = static_cast<int>(valid_count(n, C, l, t, causal));
    for (; l >= 2; --l) {
      const int vcc = static_cast<int>(valid_count(n, C, l - 1, t, causal));  // usable children level
      const int nc = warp_compact(cand, cand >= 0 && cand < vc, tmp[warp]);
      int nk = nc;
      if (nc > K && l <= ltop && l >= ltop - 2) {
        float s = lane < nc ? __ldg(drow + dense_slot0(ltop - l) + cand) : -INFINITY;
        int idx = lane < nc ? cand : INT_MAX;
        warp_sort_desc(s, idx);
        cand = idx;
        nk = K;
      } else if (nc > K) {
        // M-tile m holds candidates 8m .. 8m+7: row gid = first child, row gid + 8 = second.
        float um[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          if (8 * m >= nc) break;
          const int c = __shfl_sync(kFull, cand, 8 * m + gid);
          const bool have = 8 * m + gid < nc;
          const int64_t r0 = have ? 2 * static_cast<int64_t>(c) : 0;
          const bool has1 = have && r0 + 1 < vcc;
          const uint4* p0 = PL + (off[l - 1] + r0) * (D / 4) + tig;
          const uint4* p1 = PL + (off[l - 1] + (has1 ? r0 + 1 : r0)) * (D / 4) + tig;
          uint4 x0[D / 16], x1[D / 16];
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            x0[ks] = __ldg(p0 + 4 * ks);
            x1[ks] = __ldg(p1 + 4 * ks);
          }
          // Four accumulators (hi / lo x even / odd k step) keep the MMA
          // dependency chains short.
          float ah0[4] = {0.f, 0.f, 0.f, 0.f}, ah1[4] = {0.f, 0.f, 0.f, 0.f};
          float al0[4] = {0.f, 0.f, 0.f, 0.f}, al1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t hi[4] = {x0[ks].x, x1[ks].x, x0[ks].y, x1[ks].y};
            const uint32_t lo[4] = {x0[ks].z, x1[ks].z, x0[ks].w, x1[ks].w};
            mma_bf16((ks & 1) ? ah1 : ah0, hi, qb[ks][0], qb[ks][1]);
            mma_bf16((ks & 1) ? al1 : al0, lo, qb[ks][0], qb[ks][1]);
          }
          float acc[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = (ah0[i] + ah1[i]) + (al0[i] + al1[i]);
          // acc: [first child, head 2tig], [first, 2tig+1], [second, 2tig], [second, 2tig+1]
          float u = 0.f;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (2 * tig + j < G) {
              const float s0 = a.scale * acc[j];
              u += has1 ? lse2(s0, a.scale * acc[2 + j]) : s0;
            }
          }
          u += __shfl_xor_sync(kFull, u, 1);
          u += __shfl_xor_sync(kFull, u, 2);
          um[m] = have ? u : -INFINITY;
        }
        const int src = 4 * (lane & 7);
        const float v0 = __shfl_sync(kFull, um[0], src), v1 = __shfl_sync(kFull, um[1], src);
        const float v2 = __shfl_sync(kFull, um[2], src), v3 = __shfl_sync(kFull, um[3], src);
        const int mm = lane >> 3;
        float s = mm == 0 ? v0 : (mm == 1 ? v1 : (mm == 2 ? v2 : v3));
        int idx = lane < nc ? cand : INT_MAX;
        if (lane >= nc) s = -INFINITY;
        warp_sort_desc(s, idx);
        cand = idx;
        nk = K;
      }
      const int parent = __shfl_sync(kFull, cand, lane >> 1);
      cand = (lane >> 1) < nk ? 2 * parent + (lane & 1) : -1;
      vc = vcc;
    }
  }
  // Leaf-level candidates.
  const int nc = warp_compact(cand, cand >= 0 && cand < static_cast<int>(valid_count(n, C, 1, t, causal)), tmp[warp]);
  if (nc <= K) {
    int idx = lane < nc ? cand : INT_MAX;
    warp_sort_asc(idx);
    if (lane < K) {
      sel[row * K + lane] = idx == INT_MAX ? -1 : idx;
      if (sel_score) sel_score[row * K + lane] = nanv;
    }
    if (lane == 0) ws.ncand[row] = -1;
    return;
  }
  ws.cand[row * 32 + lane] = lane < nc ? cand : -1;
  if (lane == 0) ws.ncand[row] = nc;
  // The count's old value is the pair's place in its bucket, so the scatter
  // needs no second atomic.
  if (lane < nc)
    ws.rank[row * 32 + lane] = atomicAdd(&ws.count[(bh * ws.nwin + (i_row >> ws.win_shift)) * level_size(n, C, 1) + cand], 1);
}

// ---------------------------------------------------------------- grouping
// Exclusive scans of the pair counts (bucket offsets) and of the work items
// per bucket, by one CTA.
__global__ void __launch_bounds__(1024) scan_kernel(Ws ws, int nb) {
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
      c[j] = i < nb ? ws.count[i] : 0;
      it[j] = (c[j] + kPairsPerItem - 1) / kPairsPerItem;
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
        ws.bucket_off[i] = e0;
        ws.item_off[i] = e1;
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
    ws.bucket_off[nb] = carry[0];
    ws.item_off[nb] = carry[1];
  }
}

// One thread per (row, slot): writes each pair into its leaf's bucket. A
// pair holds the query's row index within its (b, kv head), not its position.
__global__ void __launch_bounds__(256) scatter_kernel(Ws ws, int64_t rows, int Nq, int M1) {
  const int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = x >> 5;
  const int slot = static_cast<int>(x & 31);
  if (row >= rows) return;
  const int nc = ws.ncand[row];
  if (slot >= nc) return;
  const int leaf = ws.cand[row * 32 + slot];
  const int64_t bh = row / Nq, t = row % Nq;
  const int64_t bucket = (bh * ws.nwin + (t >> ws.win_shift)) * M1 + leaf;
  const int pos = ws.rank[row * 32 + slot];
  ws.pairs[ws.bucket_off[bucket] + pos] = (static_cast<uint32_t>(t) << 5) | static_cast<uint32_t>(slot);
}

// Item -> (bucket, pair range) map: one thread per bucket writes its items' entries.
__global__ void __launch_bounds__(256) itemize_kernel(Ws ws, int nb, int M1) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nb) return;
  const int i0 = ws.item_off[b], i1 = ws.item_off[b + 1];
  const int p0 = ws.bucket_off[b], p1 = ws.bucket_off[b + 1];
  const int bh = b / (ws.nwin * M1), leaf = b % M1;  // bucket = (bh * nwin + window) * M1 + leaf
  for (int i = i0; i < i1; ++i) {
    ws.item_bucket[i] = b;
    const int lo = p0 + (i - i0) * kPairsPerItem;
    ws.item_info[i] = make_int4(bh, lo, min(lo + kPairsPerItem, p1), leaf);
  }
}

// ---------------------------------------------------------------- stage 2
// Stage 2. Work items (128 pairs of one bucket) are walked grid-strided, so
// that at any time all CTAs work on neighbouring buckets (the same query
// window). Per item the leaf's C x d key
// tile is brought into shared memory by bulk tensor copies (double buffered
// across items, reused when the next item has the same bucket). Each warp
// scores 16-row M tiles: the G heads of 16 / G queries (a query tile of
// Q_tile = 4 queries x G heads is split into passes of 16 rows), whose rows
// arrive as one 3-D tensor box per query (heads x d) in a per-warp double
// buffer. Both MMA operands are read with ldmatrix from 128-byte swizzled
// boxes. Per (query, head) row: LSE over the usable keys of the leaf; then
// the sum over the G heads of each query.
template <int D, int G, int CC>
__global__ void __launch_bounds__(kLeafThreads, 2)
    leaf_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk, PrefillArgs a,
                Ws ws, int nb, int M1, unsigned long long* faults) {
  constexpr int kNT = CC / 8;                  // 8-key N tiles per leaf
  constexpr int kKS = D / 16;                  // 16-wide k steps
  constexpr int kBoxes = D / 64;               // 64-column boxes per row
  constexpr int kP = G >= 8 ? 2 : kQTile;      // queries per 16-row M tile
  constexpr int kSlot = 1024;                  // one query's G rows of one box, 1 KB aligned
  constexpr int kQStage = kP * kBoxes * kSlot;
  constexpr int kKeyBytes = CC * D * 2;
  constexpr int kWarps = kLeafThreads / 32;
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t kbar[2];
  __shared__ uint64_t qbar[kWarps][2];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  unsigned char* qring = smem + 2 * kKeyBytes + warp * 2 * kQStage;
  const bool causal = a.causal != 0;
  const float sl2 = a.scale * kLog2e;
  if (threadIdx.x == 0) {
    mbar_init(&kbar[0], 1);
    mbar_init(&kbar[1], 1);
  }
  if (lane == 0) {
    mbar_init(&qbar[warp][0], 1);
    mbar_init(&qbar[warp][1], 1);
  }
  mbar_init_fence();
  __syncthreads();

  const int total = ws.item_off[nb];
  int item = blockIdx.x;
  if (item >= total) return;
  const int64_t bucket_span = static_cast<int64_t>(ws.nwin) * M1;  // buckets per (b, kv head)
  auto issue_key = [&](int bk, int bf) {  // thread 0 only
    const int64_t bhh = bk / bucket_span, leaf = bk % M1;
    const int y = static_cast<int>(bhh * a.N + leaf * CC);
    fence_proxy_async();
    mbar_expect_tx(&kbar[bf], kKeyBytes);
#pragma unroll
    for (int x = 0; x < kBoxes; ++x) tma_load_2d(smem + bf * kKeyBytes + x * CC * 128, &tmk, 64 * x, y, &kbar[bf]);
  };
  int bucket = ws.item_bucket[item];
  int buf = 0;
  uint32_t kph = 0, kpend = 1;  // parity and pending-load bits per key buffer
  if (threadIdx.x == 0) issue_key(bucket, 0);
  int qst = 0;
  uint32_t qph = 0;

  while (true) {
    const int p_lo = ws.bucket_off[bucket] + (item - ws.item_off[bucket]) * kPairsPerItem;
    const int p_hi = min(p_lo + kPairsPerItem, ws.bucket_off[bucket + 1]);
    const int next_item = item + gridDim.x;
    const int next = next_item < total ? ws.item_bucket[next_item] : -1;
    if (next >= 0 && next != bucket) {
      if (threadIdx.x == 0) issue_key(next, buf ^ 1);
      kpend |= 1u << (buf ^ 1);
    }
    if (kpend & (1u << buf)) {
      mbar_wait(&kbar[buf], (kph >> buf) & 1u, faults);
      kph ^= 1u << buf;
      kpend &= ~(1u << buf);
    }
    const unsigned char* tile = smem + buf * kKeyBytes;
    const int64_t bh = bucket / bucket_span;
    const int64_t key0 = static_cast<int64_t>(bucket % M1) * CC;
    const int nkeys = static_cast<int>(min(static_cast<int64_t>(CC), a.N - key0));
    const int64_t b = bh / a.H_kv, h = bh % a.H_kv;
    const int zq = static_cast<int>(b * a.H_q + h * G);
    const int nunits = (p_hi - p_lo + kP - 1) / kP;

    // Queries of unit u into q stage st (lane 0 issues; one box per query per 64 columns).
    auto issue_q = [&](int u, int st) {
      if (lane == 0) {
        const int pu = p_lo + u * kP;
        const int nv = min(kP, p_hi - pu);
        unsigned char* qs = qring + st * kQStage;
        fence_proxy_async();
        mbar_expect_tx(&qbar[warp][st], static_cast<uint32_t>(nv * G * D * 2));
        for (int i = 0; i < nv; ++i) {
          const int tq = static_cast<int>(ws.pairs[pu + i] >> 5);
#pragma unroll
          for (int x = 0; x < kBoxes; ++x)
            tma_load_3d(qs + x * kP * kSlot + i * kSlot, &tmq, 64 * x, tq, zq, &qbar[warp][st]);
        }
      }
    };
    int u = warp;
    if (u < nunits) issue_q(u, qst);
    for (; u < nunits; u += kWarps) {
      const int un = u + kWarps;
      if (un < nunits) issue_q(un, qst ^ 1);
      mbar_wait(&qbar[warp][qst], (qph >> qst) & 1u, faults);
      qph ^= 1u << qst;
      const unsigned char* qs = qring + qst * kQStage;

      const int pu = p_lo + u * kP;
      const uint32_t pw = (lane < kP && pu + lane < p_hi) ? ws.pairs[pu + lane] : 0xffffffffu;
      int nvk[2];
      bool ok[2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = gid + 8 * half;
        const int pi = r / G;
        const uint32_t w = __shfl_sync(kFull, pw, pi < kP ? pi : 0);
        ok[half] = pi < kP && w != 0xffffffffu;
        const int64_t tq = ok[half] ? a.q0 + static_cast<int64_t>(w >> 5) : 0;  // query position
        int64_t nv = nkeys;
        if (causal) nv = min(nv, tq - key0 + 1);
        nvk[half] = static_cast<int>(max(nv, static_cast<int64_t>(0)));
      }
      // A (query rows) and B (keys) fragments via ldmatrix.
      const int mat = lane >> 3, mr = lane & 7;
      const int arow = mr + 8 * (mat & 1);                 // M-tile row this lane addresses
      const int ap = arow / G < kP ? arow / G : 0, ag = arow % G;
      const unsigned char* abase = qs + ap * kSlot + ag * 128;
      float acc[kNT][4];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks) {
        uint32_t af[4];
        {
          const int col = 16 * ks + 8 * (mat >> 1);
          const int bx = col >> 6, c16 = (col & 63) >> 3;
          ldsm_x4(af, abase + bx * kP * kSlot + ((c16 ^ (ag & 7)) << 4));
        }
#pragma unroll
        for (int nt = 0; nt < kNT; nt += 2) {
          uint32_t bf[4];
          const int krow = 8 * (nt + (mat >> 1)) + mr;
          ldsm_x4(bf, tile + swz128<CC>(krow, 16 * ks + 8 * (mat & 1)));
          mma_bf16(acc[nt], af, bf[0], bf[1]);
          mma_bf16(acc[nt + 1], af, bf[2], bf[3]);
        }
      }
      __syncwarp();  // the stage is refilled two units later
      // Per (query, head) row: LSE over the usable keys, in log2 units.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int nv = nvk[half];
        float mx = -INFINITY;
        if (nv >= CC) {
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) mx = fmaxf(mx, fmaxf(acc[nt][2 * half], acc[nt][2 * half + 1]));
        } else {
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e)
              if (8 * nt + 2 * tig + e < nv) mx = fmaxf(mx, acc[nt][2 * half + e]);
        }
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const float mxs = mx * sl2;
        float sum = 0.f;
        if (nv >= CC) {
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) sum += exp2f(fmaf(acc[nt][2 * half + e], sl2, -mxs));
        } else {
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e)
              if (8 * nt + 2 * tig + e < nv) sum += exp2f(fmaf(acc[nt][2 * half + e], sl2, -mxs));
        }
        sum += __shfl_xor_sync(kFull, sum, 1);
        sum += __shfl_xor_sync(kFull, sum, 2);
        float uu = ok[half] ? mx * a.scale + logf(sum) : 0.f;
        // Sum over the G heads of each query: rows r .. r + G - 1 sit in
        // lanes that differ in the low log2(G) bits of gid.
#pragma unroll
        for (int o = 4; o < 4 * G; o <<= 1) uu += __shfl_xor_sync(kFull, uu, o);
        const int r = gid + 8 * half;
        const int pi = r / G;
        const uint32_t w = __shfl_sync(kFull, pw, pi < kP ? pi : 0);
        if (tig == 0 && (gid % G) == 0 && ok[half]) {
          const int64_t orow = bh * a.Nq + static_cast<int64_t>(w >> 5);
          ws.score[orow * 32 + (w & 31)] = uu;
        }
      }
      qst ^= 1;
    }
    __syncthreads();  // every warp is done with the key tile (and its query stages)
    if (next < 0) break;
    if (next != bucket) buf ^= 1;
    bucket = next;
    item = next_item;
  }
}

// ---------------------------------------------------------------- final top-K
__global__ void __launch_bounds__(256) final_kernel(PrefillArgs a, Ws ws, int32_t* __restrict__ sel,
                                                    float* __restrict__ sel_score, int64_t rows) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= rows) return;
  const int nc = ws.ncand[row];
  if (nc < 0) return;  // stage 1 kept every usable leaf unscored and wrote sel
  float s = lane < nc ? ws.score[row * 32 + lane] : -INFINITY;
  int idx = lane < nc ? ws.cand[row * 32 + lane] : INT_MAX;
  // Top K (K <= 16) by (score descending, index ascending): the first four
  // phases of a 32-lane bitonic sort order lanes 0..15 best-first and lanes
  // 16..31 worst-first; keeping the better of lanes i and i + 16 leaves the 16
  // best in lanes 0..15. Only for K < 16 are those 16 then ordered, so that
  // lanes 0..K-1 hold the K best.
  auto cmpx = [&](int j, bool keep_best) {
    const float os = __shfl_xor_sync(kFull, s, j);
    const int oi = __shfl_xor_sync(kFull, idx, j);
    if (keep_best ? ranks_before(os, oi, s, idx) : ranks_before(s, idx, os, oi)) {
      s = os;
      idx = oi;
    }
  };
#pragma unroll
  for (int k = 2; k <= 16; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) cmpx(j, ((lane & k) == 0) == ((lane & j) == 0));
  cmpx(16, (lane & 16) == 0);
  if (a.K < 16) {
#pragma unroll
    for (int j = 8; j > 0; j >>= 1) cmpx(j, (lane & j) == 0);
  }
  if (lane >= a.K) {
    idx = INT_MAX;
    s = 0.f;
  }
  // The K kept pairs ascending by index: a 16-lane bitonic sort (lanes 16..31
  // hold only empty slots and take no part).
#pragma unroll
  for (int k = 2; k <= 16; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int oi = __shfl_xor_sync(kFull, idx, j);
      const float os = __shfl_xor_sync(kFull, s, j);
      const bool keep_small = ((lane & k) == 0) == ((lane & j) == 0);
      if (keep_small ? (oi < idx) : (oi > idx)) {
        idx = oi;
        s = os;
      }
    }
  }
  if (lane < a.K) {
    sel[row * a.K + lane] = idx;
    if (sel_score) sel_score[row * a.K + lane] = s;
  }
}

int sm_count() {
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

size_t select2_workspace_bytes(const PrefillArgs& a) { return carve(a, nullptr, nullptr); }

cudaError_t launch_select2(const PrefillArgs& a, const void* q, const void* k, const float* pyr, const Layout& lay,
                           int32_t* sel, float* sel_score, void* ws_ptr, cudaStream_t st) {
  Ws ws;
  carve(a, static_cast<char*>(ws_ptr), &ws);
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * a.Nq;
  const int M1 = static_cast<int>(level_size(a.N, a.C, 1));
  const int nb = a.B * a.H_kv * ws.nwin * M1;
  cudaError_t e = cudaMemsetAsync(ws.count, 0, static_cast<size_t>(nb) * 4, st);
  if (e != cudaSuccess) return e;
  const int G = a.H_q / a.H_kv;
  {
    const int64_t n4 = static_cast<int64_t>(a.B) * a.H_kv * lay.R * a.d / 4;
    const int64_t gb = (n4 + 255) / 256;
    const unsigned g = static_cast<unsigned>(gb < sm_count() * 16 ? gb : sm_count() * 16);
    TimedLaunch tl("split_kernel", st);
    split_kernel<<<g, 256, 0, st>>>(reinterpret_cast<const float4*>(pyr), ws.planes, reinterpret_cast<uint2*>(ws.hi),
                                    reinterpret_cast<uint2*>(ws.lo), n4);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (ws.dense && (e = launch_router_top(a, q, lay, ws, st)) != cudaSuccess) return e;
  e = dispatch_tdg(PISA_DTYPE_BF16, a.d, G, [&](auto, auto dd, auto gg) -> cudaError_t {
    constexpr int D = decltype(dd)::value, GG = decltype(gg)::value;
    TimedLaunch tl("router_kernel", st);
    router_kernel<D, GG><<<static_cast<unsigned>((rows + kRouterWarps - 1) / kRouterWarps), kRouterWarps * 32, 0,
                           st>>>(static_cast<const bf16*>(q), pyr, lay, a, ws, sel, sel_score);
    count_launch();
    return cudaGetLastError();
  });
  if (e != cudaSuccess) return e;
  {
    TimedLaunch tl("scan_kernel", st);
    scan_kernel<<<1, 1024, 0, st>>>(ws, nb);
  }
  count_launch();
  {
    TimedLaunch tl("scatter_kernel", st);
    scatter_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(ws, rows, a.Nq, M1);
  }
  count_launch();
  {
    TimedLaunch tl("itemize_kernel", st);
    itemize_kernel<<<static_cast<unsigned>((nb + 255) / 256), 256, 0, st>>>(ws, nb, M1);
  }
  count_launch();
  if (leaf_umma_supported(a)) {
    if ((e = launch_leaf_umma(a, q, k, ws, nb, M1, st)) != cudaSuccess) return e;
  } else {
    CUtensorMap tmq, tmk;
    const int G0 = a.H_q / a.H_kv;
    e = make_tmap_bf16_3d(&tmq, q, a.d, a.Nq, static_cast<uint64_t>(a.B) * a.H_q, 1, G0);
    if (e == cudaSuccess) e = make_tmap_bf16_2d(&tmk, k, a.d, static_cast<uint64_t>(a.B) * a.H_kv * a.N, a.C);
    if (e != cudaSuccess) return e;
    unsigned long long* faults = wait_fault_counter();
    e = dispatch_tdg(PISA_DTYPE_BF16, a.d, G, [&](auto, auto dd, auto gg) -> cudaError_t {
      constexpr int D = decltype(dd)::value, GG = decltype(gg)::value;
      constexpr int kP = GG >= 8 ? 2 : kQTile;
      const size_t qstage = static_cast<size_t>(kP) * (D / 64) * 1024;
      auto launch = [&](auto kern, int CC) -> cudaError_t {
        const size_t smem = 2 * static_cast<size_t>(CC) * D * 2 + (kLeafThreads / 32) * 2 * qstage + 1024;
        cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e2 != cudaSuccess) return e2;
        int per_sm = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLeafThreads, smem) != cudaSuccess ||
            per_sm < 1)
          per_sm = 1;
        TimedLaunch tl("leaf_kernel", st);
        kern<<<static_cast<unsigned>(sm_count() * per_sm), kLeafThreads, smem, st>>>(tmq, tmk, a, ws, nb, M1, faults);
        count_launch();
        return cudaGetLastError();
      };
      return a.C == 64 ? launch(leaf_kernel<D, GG, 64>, 64) : launch(leaf_kernel<D, GG, 32>, 32);
    });
    if (e != cudaSuccess) return e;
  }
  {
    TimedLaunch tl("final_kernel", st);
    final_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(a, ws, sel, sel_score, rows);
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace pisa
