// Stage-2 leaf scorer on the fifth-generation tensor cores (tcgen05) for
// groups of G_Q = 8 query heads, d = 128, C = 64 (the paper's kernel
// design, §Kernels: a d x C key tile reused across a (Q_tile G_Q) x d query
// tile).
//
// One CTA per SM runs a warp-specialised pipeline over the stage-2 work
// items (64 (query, leaf) pairs of one bucket, walked grid-strided so that
// all SMs work in the current query window):
//   warps 8-11 (loads): per tile of 16 queries, their 8 head rows
//     (16 x 8 = 128 rows) gathered with 16-byte cp.async straight into the
//     swizzled operand layout of a ring of query stages, running ahead of the
//     MMAs (many small bulk copies cost more than one per 2 KB row group);
//   warp 12, one lane (MMA): per item, the leaf's 64 x 128 key tile by bulk
//     tensor copy, issued one item ahead into a double buffer; per tile, eight
//     tcgen05.mma (M = 128 query-head
//     rows, N = 64 keys, K = 16 each) into a ring of TMEM accumulators,
//     then tcgen05.commit to release the query stage (and, after an item's
//     last tile, the key tile) and to publish the accumulator;
//   warps 0-7 (epilogue): two groups of four warps take alternate tiles;
//     warp w reads TMEM lane quarter w & 3, each thread owns one lane = one
//     (query, head) row and loads its 64 key scores with tcgen05.ld, takes the
//     max and exp-sum over its usable keys into the row's LSE, the 8 heads of
//     a query are summed with three shuffles, and one lane per query stores
//     the leaf score.
// Operands sit in shared memory as 128-byte-swizzled K-major tiles (rows of
// 64 bf16, 8-row groups 1 KB apart), which is both the bulk-copy layout and
// the MMA descriptor layout. Every mbarrier wait is bounded in time; the
// TMEM allocation is always released before exit.
#include "dispatch.cuh"
#include "select2_ws.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace pisa {

namespace {

constexpr int kEpiGroups = 2;              // epilogue warp groups, taking alternate tiles
constexpr int kEpiWarps = 4 * kEpiGroups;  // warps 0 .. kEpiWarps - 1
constexpr int kLoadWarps = 4;              // warps 8-11 gather the query rows
constexpr int kMmaWarp = kEpiWarps + kLoadWarps;  // warp 12 issues the MMAs
constexpr int kUmmaThreads = 32 * (kMmaWarp + 1);
constexpr int kLoaders = 32 * kLoadWarps;
constexpr int kTilePairs = 16;             // queries per MMA tile (x 8 heads = 128 rows)
constexpr int kQStages = 5;
constexpr int kQStageBytes = kTilePairs * 8 * 128 * 2;  // 16 queries x 8 heads x 256 B = 32 KB (two 64-col halves)
constexpr int kKeyBytes = 64 * 128 * 2;                 // 16 KB (two 64-col halves)
constexpr int kAccCols = 64;                            // fp32 columns per accumulator (N = 64 keys)
constexpr int kAccStages = 4;                           // TMEM accumulator buffers
constexpr uint32_t kTmemCols = kAccStages * kAccCols;

struct Cursor2 {
  int item, bh, leaf, p_lo, p_hi, ntiles;
};

__global__ void __launch_bounds__(kUmmaThreads, 1)
    leaf_umma_kernel(const bf16* __restrict__ q, const __grid_constant__ CUtensorMap tmk, PrefillArgs a, Ws ws,
                     int nb, int M1, unsigned long long* faults) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t kfull[2], kempty[2], qfull[kQStages], qempty[kQStages], accfull[kAccStages], accempty[kAccStages];
  __shared__ uint32_t tmem_base_sh;
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* kbuf = smem;                       // [2][kKeyBytes]
  unsigned char* qbuf = smem + 2 * kKeyBytes;       // [kQStages][kQStageBytes]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < kAccStages; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 4);  // the four warps of the group that owns the tile
    }
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&qfull[i], kLoaders);
      mbar_init(&qempty[i], 1);
    }
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  const int total = ws.item_off[nb];
  const bool causal = a.causal != 0;
  // Work-item records are loaded one item ahead (one 16-byte load each).
  auto info = [&](int item) { return item < total ? ws.item_info[item] : make_int4(0, 0, 0, 0); };
  auto cursor = [&](int item, int4 inf) {
    Cursor2 c;
    c.item = item;
    c.bh = inf.x;
    c.leaf = inf.w;
    c.p_lo = inf.y;
    c.p_hi = inf.z;
    c.ntiles = (c.p_hi - c.p_lo + kTilePairs - 1) / kTilePairs;
    return c;
  };
  // Position in this CTA's stream of tiles: items blockIdx.x, + gridDim.x,
  // ..., each cut into tiles of kTilePairs pairs.
  struct Stream {
    int item, tl;
    Cursor2 c;
    int4 inf_next;
  };
  auto stream_begin = [&]() {
    Stream st;
    st.item = blockIdx.x;
    st.tl = 0;
    st.c = cursor(st.item, info(st.item));
    st.inf_next = info(st.item + gridDim.x);
    return st;
  };
  auto stream_next = [&](Stream st) {
    if (st.item < total && ++st.tl >= st.c.ntiles) {
      st.item += gridDim.x;
      st.tl = 0;
      if (st.item < total) {
        st.c = cursor(st.item, st.inf_next);
        st.inf_next = info(st.item + gridDim.x);
      }
    }
    return st;
  };

  if (warp >= kEpiWarps && warp < kMmaWarp) {
    // ---------------------------------------------------------- loads
    const int lw = warp - kEpiWarps;              // loader warp 0..kLoadWarps-1
    const int jcol = lane & 15;                   // 16-byte column of a 256-byte query row
    const int g0 = 2 * lw + (lane >> 4);          // head row g0 (and g0 + 4 with two loader warps)
    const int64_t head_stride = static_cast<int64_t>(a.Nq) * 128;
    int nq = 0;                        // uses of the query ring so far
    // Each tile's pair words are loaded one tile ahead, so their latency
    // hides behind the previous tile's copies.
    auto tile_words = [&](const Stream& st) -> uint32_t {
      if (st.item >= total) return 0u;
      const int p0 = st.c.p_lo + st.tl * kTilePairs;
      return lane < min(kTilePairs, st.c.p_hi - p0) ? ws.pairs[p0 + lane] : 0u;
    };
    Stream sm = stream_begin();
    uint32_t tw_next = tile_words(sm);
    while (sm.item < total) {
      const Stream cur = sm;
      const uint32_t twv = tw_next;
      sm = stream_next(sm);
      tw_next = tile_words(sm);
      const Cursor2& c = cur.c;
      const int64_t b = c.bh / a.H_kv, h = c.bh % a.H_kv;
      const bf16* qg = q + (b * a.H_q + h * 8) * head_stride;  // head 0 of the group
      const bf16* qrow0 = qg + g0 * head_stride + jcol * 8;   // this thread's column of head g0
      {
        const int qs = nq % kQStages;
        const int p0 = c.p_lo + cur.tl * kTilePairs;
        const int np = min(kTilePairs, c.p_hi - p0);
        // Loader thread (warp lw, lane l): 16-byte column j = l & 15 of head
        // row g0 = 2 lw + (l >> 4) (and g0 + 4 with two loader warps) of every query of the tile,
        // so each copy instruction moves two whole 256-byte rows. The tile's
        // query rows are read once per warp and shared by shuffle.
        const int tw = static_cast<int>(twv >> 5);
        mbar_wait(&qempty[qs], ((nq / kQStages) & 1) ^ 1, faults);
        const uint32_t qd = smem_u32(qbuf + qs * kQStageBytes);
        const uint32_t d0 = qd + (jcol >> 3) * (kQStageBytes / 2) + g0 * 128 + (((jcol & 7) ^ g0) << 4);
        // Unrolled over the tile's 16 slots so that the shuffles and copies
        // of different slots overlap instead of forming one chain.
        int tq[kTilePairs];
#pragma unroll
        for (int i = 0; i < kTilePairs; ++i) tq[i] = __shfl_sync(kFull, tw, i);
#pragma unroll
        for (int i = 0; i < kTilePairs; ++i) {
          if (i < np) {
            const bf16* src = qrow0 + static_cast<int64_t>(tq[i]) * 128;
            cp16(d0 + i * 1024, src);
            if (kLoadWarps == 2) {
              const uint32_t d1 =
                  qd + (jcol >> 3) * (kQStageBytes / 2) + (g0 + 4) * 128 + (((jcol & 7) ^ (g0 + 4)) << 4);
              cp16(d1 + i * 1024, src + 4 * head_stride);
            }
          }
        }
        // The stage's barrier completes once every loader thread's copies so
        // far have landed; the MMA thread fences the async proxy after
        // waiting on it. The loader itself never waits for its copies.
        cp_arrive_noinc(&qfull[qs]);
        ++nq;
      }
    }
    cp_wait<0>();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      int nk = 0, nq = 0, na = 0;
      // Key tiles are loaded by this thread one item ahead; a key buffer is
      // refilled only after this thread's own commit of its last MMAs.
      auto load_key = [&](int4 ki, int n) {
        const int kbn = n & 1;
        mbar_wait(&kempty[kbn], ((n >> 1) & 1) ^ 1, faults);
        const int ky = static_cast<int>(static_cast<int64_t>(ki.x) * a.N + static_cast<int64_t>(ki.w) * 64);
        fence_proxy_async();
        mbar_expect_tx(&kfull[kbn], kKeyBytes);
        tma_load_2d(kbuf + kbn * kKeyBytes, &tmk, 0, ky, &kfull[kbn]);
        tma_load_2d(kbuf + kbn * kKeyBytes + 64 * 128, &tmk, 64, ky, &kfull[kbn]);
      };
      int4 inf = info(blockIdx.x);
      if (blockIdx.x < total) load_key(inf, 0);
      for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const Cursor2 c = cursor(item, inf);
        inf = info(item + gridDim.x);
        if (item + gridDim.x < total) load_key(inf, nk + 1);
        const int kb = nk & 1;
        mbar_wait(&kfull[kb], (nk >> 1) & 1, faults);
        const uint32_t ka = smem_u32(kbuf + kb * kKeyBytes);
        for (int tl = 0; tl < c.ntiles; ++tl) {
          const int qs = nq % kQStages;
          mbar_wait(&qfull[qs], (nq / kQStages) & 1, faults);
          fence_proxy_async();  // the loaders' cp.async writes, before the tensor cores read them
          const int as = na % kAccStages;
          mbar_wait(&accempty[as], ((na / kAccStages) & 1) ^ 1, faults);
          tc_fence_after();
          const uint32_t qa = smem_u32(qbuf + qs * kQStageBytes);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks >> 2) * (kQStageBytes / 2) + (ks & 3) * 32;
            const uint32_t koff = (ks >> 2) * (64 * 128) + (ks & 3) * 32;
            umma_bf16(tmem + as * kAccCols, sw128_desc(qa + off), sw128_desc(ka + koff), kIdesc, ks > 0);
          }
          umma_commit(&qempty[qs]);
          umma_commit(&accfull[as]);
          ++nq;
          ++na;
        }
        umma_commit(&kempty[kb]);
        ++nk;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // Warps 0-3 take the even tiles of the stream and warps 4-7 the odd
    // ones, so the two groups overlap one tile's TMEM load and barrier waits
    // with the other's exponentials. Warp w of a group reads TMEM lane
    // quarter w & 3; each thread owns one (query, head) row and all 64 of
    // its key scores.
    const float sl2 = a.scale * 1.4426950408889634f;
    const int qtr = warp & 3, grp = warp >> 2;
    const int row = 32 * qtr + lane;  // TMEM lane = (query, head) row of the tile
    // This group's tiles are every other tile of the stream; each one's pair
    // word is loaded one own tile ahead.
    auto row_word = [&](const Stream& st) -> uint32_t {
      if (st.item >= total) return 0xffffffffu;
      const int p = st.c.p_lo + st.tl * kTilePairs + row / 8;
      return p < st.c.p_hi ? ws.pairs[p] : 0xffffffffu;
    };
    Stream sm = stream_begin();
    int na = 0;
    if (grp == 1) {
      sm = stream_next(sm);
      na = 1;
    }
    uint32_t w_next = row_word(sm);
    while (sm.item < total) {
      const Cursor2 c = sm.c;
      const uint32_t w = w_next;
      const int na_cur = na;
      sm = stream_next(stream_next(sm));
      na += 2;
      w_next = row_word(sm);
      {
        const bool ok = w != 0xffffffffu;
        const int64_t key0 = static_cast<int64_t>(c.leaf) * 64;
        int nv = static_cast<int>(min(static_cast<int64_t>(64), a.N - key0));
        if (causal && ok)  // the pair holds the query's row; its position is q0 + row
          nv = static_cast<int>(min(static_cast<int64_t>(nv), a.q0 + static_cast<int64_t>(w >> 5) - key0 + 1));
        const int as = na_cur % kAccStages;
        mbar_wait(&accfull[as], (na_cur / kAccStages) & 1, faults);
        __syncwarp();  // the TMEM load below is warp-collective
        tc_fence_after();
        uint32_t v[kAccCols];
        tmem_ld_cols<kAccCols>(tmem + (static_cast<uint32_t>(32 * qtr) << 16) + as * kAccCols, v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[as]);
        // Max and sum of exponentials over the usable keys (four chains each).
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (nv >= kAccCols) {
#pragma unroll
          for (int j = 0; j < kAccCols; ++j) m4[j & 3] = fmaxf(m4[j & 3], __uint_as_float(v[j]));
        } else {
#pragma unroll
          for (int j = 0; j < kAccCols; ++j)
            if (j < nv) m4[j & 3] = fmaxf(m4[j & 3], __uint_as_float(v[j]));
        }
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        const float mxs = mx * sl2;
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        if (nv >= kAccCols) {
#pragma unroll
          for (int j = 0; j < kAccCols; ++j) s4[j & 3] += ex2_approx(fmaf(__uint_as_float(v[j]), sl2, -mxs));
        } else {
#pragma unroll
          for (int j = 0; j < kAccCols; ++j)
            if (j < nv) s4[j & 3] += ex2_approx(fmaf(__uint_as_float(v[j]), sl2, -mxs));
        }
        const float z = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        float u = ok && nv > 0 ? mx * a.scale + logf(z) : 0.f;
        u += __shfl_xor_sync(kFull, u, 1);
        u += __shfl_xor_sync(kFull, u, 2);
        u += __shfl_xor_sync(kFull, u, 4);
        if (ok && (row & 7) == 0) {
          const int64_t orow = static_cast<int64_t>(c.bh) * a.Nq + static_cast<int64_t>(w >> 5);
          ws.score[orow * 32 + (w & 31)] = u;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

int sm_count_umma() {
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

bool leaf_umma_supported(const PrefillArgs& a) {
  return a.dtype == PISA_DTYPE_BF16 && a.d == 128 && a.C == 64 && a.H_q == 8 * a.H_kv;
}

cudaError_t launch_leaf_umma(const PrefillArgs& a, const void* q, const void* k, const Ws& ws, int nb, int M1,
                             cudaStream_t st) {
  CUtensorMap tmk;
  cudaError_t e = make_tmap_bf16_2d(&tmk, k, a.d, static_cast<uint64_t>(a.B) * a.H_kv * a.N, 64);
  if (e != cudaSuccess) return e;
  const size_t smem = 2 * static_cast<size_t>(kKeyBytes) + kQStages * static_cast<size_t>(kQStageBytes) + 1024;
  e = cudaFuncSetAttribute(leaf_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  TimedLaunch tl("leaf_umma_kernel", st);
  leaf_umma_kernel<<<static_cast<unsigned>(sm_count_umma()), kUmmaThreads, smem, st>>>(
      static_cast<const bf16*>(q), tmk, a, ws, nb, M1, wait_fault_counter());
  count_launch();
  return cudaGetLastError();
}

}  // namespace pisa
