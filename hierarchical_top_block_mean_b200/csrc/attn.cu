// Block-sparse attention forward for bf16 prefill (paper §BSA):
//   o_t = sum_{j in T_t} exp(scale q_t.k_j) v_j / sum_{j in T_t} exp(scale q_t.k_j)
// over the raw keys of the selected leaf blocks, for the G query heads of a
// group at once.
//
// Each warp owns one (kv head, query) row at a time and streams the row's
// selected blocks through its own ring of kAttnStages shared-memory stages,
// in chunks of kKeysPerChunk keys (K and V rows), kAttnStages - 1 chunks in
// flight while one is in use. One lane issues the chunk as
// bulk tensor copies (TMA: chunk-row x 64-column boxes with the hardware
// 128-byte swizzle) that complete on the stage's mbarrier, so the copy costs
// the warp a handful of instructions and ldmatrix reads are conflict-free.
// Per chunk:
//   S^T [chunk keys x 8 heads] = K . Q^T  (A = K via ldmatrix)
//   online softmax per head (column)
//   O^T [d x 8 heads]    += V^T . P^T       (A = V^T via ldmatrix.trans,
//                                            B = P^T via movmatrix)
// Warps are persistent and the ring runs across row boundaries, so the next
// row's first chunk is already in flight when a row finishes.
#include "attn_mma.cuh"
#include "dispatch.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace pisa {

namespace {

constexpr int kAttnWarps = 14;
constexpr int kAttnStages = 2;
constexpr int kKeysPerChunk = 16;
constexpr float kLazy = 8.f;  // headroom of the lazily moved softmax maximum (natural-log units)

// Work cursor of one warp: row, the row's selected blocks (compacted, one
// per lane, held in a register), position in that list and chunk.
struct Cursor {
  int64_t row;  // -1: exhausted
  int bh, t;    // row = bh * Nq + t: t is the query's row, q0 + t its position (divided once per row)
  int blk_lane; // this lane's entry of the row's compacted block list
  int nblk;     // blocks in the list
  int idx;      // position in the list
  int half;     // chunk within the block
};

template <int D, int CC, int G>
__global__ void __launch_bounds__(kAttnWarps * 32, 1)
    attn_kernel(const bf16* __restrict__ q, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const int32_t* __restrict__ sel, PrefillArgs a,
                bf16* __restrict__ out, float* __restrict__ lse, unsigned long long* faults) {
  constexpr int kKS = D / 16;                  // k steps of S^T; d tiles of O^T
  constexpr int kChunkBytes = kKeysPerChunk * D * 2;
  constexpr int kHalves = CC / kKeysPerChunk;  // chunks per leaf block
  constexpr int kMT = kKeysPerChunk / 16;      // 16-key M tiles per chunk
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t bars[kAttnWarps][kAttnStages];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  // 128-byte swizzled boxes need 1 KB alignment.
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem + warp * (kAttnStages * 2 * kChunkBytes);  // [stage][K|V][chunk]
  if (lane == 0) {
    for (int i = 0; i < kAttnStages; ++i) mbar_init(&bars[warp][i], 1);
    mbar_init_fence();
  }
  __syncwarp();
  uint32_t phase = 0;  // parity bit of each stage's next completion
  const int64_t n = a.N, nq = a.Nq;
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * nq;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kAttnWarps;
  const bool causal = a.causal != 0;

  // Loads row r's selection into lanes (compacted: valid blocks first).
  auto load_row = [&](int64_t r) -> Cursor {
    for (; r < rows; r += stride) {
      int b = lane < a.K ? sel[r * a.K + lane] : -1;
      const unsigned m = __ballot_sync(kFull, b >= 0);
      if (m == 0) continue;
      int out_b = b;
      if ((m & (m + 1u)) != 0u) {  // not already a prefix: compact, lane j takes the j-th valid entry
        out_b = -1;
        for (int j = 0, src = 0; j < 32; ++j) {
          const int bj = __shfl_sync(kFull, b, j);
          if ((m >> j) & 1u) {
            if (lane == src) out_b = bj;
            ++src;
          }
        }
      }
      return Cursor{r, static_cast<int>(r / nq), static_cast<int>(r % nq), out_b, __popc(m), 0, 0};
    }
    return Cursor{-1, 0, 0, -1, 0, 0, 0};
  };
  auto advance = [&](const Cursor& c) -> Cursor {
    if (c.row < 0) return c;
    if (c.half + 1 < kHalves) return Cursor{c.row, c.bh, c.t, c.blk_lane, c.nblk, c.idx, c.half + 1};
    if (c.idx + 1 < c.nblk) return Cursor{c.row, c.bh, c.t, c.blk_lane, c.nblk, c.idx + 1, 0};
    return load_row(c.row + stride);
  };
  // Issues chunk c into ring stage st: K and V rows [key0, key0 + 32) of
  // this head as 64-column boxes. Rows past the sequence or the causal limit
  // are loaded but masked; rows past the whole tensor read as zero.
  auto issue = [&](const Cursor& c, int st) {
    if (c.row < 0) return;
    const int blk = __shfl_sync(kFull, c.blk_lane, c.idx);
    if (lane == 0) {
      const int y = static_cast<int>(c.bh * n + static_cast<int64_t>(blk) * CC + c.half * kKeysPerChunk);
      unsigned char* ks = ring + st * 2 * kChunkBytes;
      unsigned char* vs = ks + kChunkBytes;
      fence_proxy_async();  // the stage's previous contents were read by ldmatrix
      mbar_expect_tx(&bars[warp][st], 2 * kChunkBytes);
#pragma unroll
      for (int x = 0; x < D; x += 64) {
        tma_load_2d(ks + x * kKeysPerChunk * 2, &tmk, x, y, &bars[warp][st]);
        tma_load_2d(vs + x * kKeysPerChunk * 2, &tmv, x, y, &bars[warp][st]);
      }
    }
  };

  // Chunks are issued in order, chunk c into stage c mod kAttnStages; tail is
  // the last one issued.
  Cursor cur = load_row(static_cast<int64_t>(blockIdx.x) * kAttnWarps + warp);
  issue(cur, 0);
  Cursor tail = cur;
#pragma unroll
  for (int i = 1; i < kAttnStages - 1; ++i) {
    tail = advance(tail);
    issue(tail, i);
  }
  int st = 0;
  int64_t row_now = -1;
  uint32_t qb[kKS][2];
  float m[2], l[2], o[kKS][4];
  int hb = 0, hh = 0;  // batch and kv head of the current row

  while (cur.row >= 0) {
    const Cursor nxt = advance(cur);
    tail = kAttnStages == 2 ? nxt : advance(tail);
    issue(tail, st == 0 ? kAttnStages - 1 : st - 1);  // the stage read in the previous iteration
    mbar_wait(&bars[warp][st], (phase >> st) & 1u, faults);
    phase ^= 1u << st;

    const int64_t t = cur.t;
    if (cur.row != row_now) {  // first chunk of a row: queries and softmax state
      hb = cur.bh / a.H_kv;
      hh = cur.bh % a.H_kv;
      row_now = cur.row;
      const bf16* qp = q + ((static_cast<int64_t>(hb) * a.H_q + hh * G + (gid < G ? gid : 0)) * nq + t) * D + 2 * tig;
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks) {
        qb[ks][0] = gid < G ? *reinterpret_cast<const uint32_t*>(qp + 16 * ks) : 0u;
        qb[ks][1] = gid < G ? *reinterpret_cast<const uint32_t*>(qp + 16 * ks + 8) : 0u;
      }
      m[0] = m[1] = -INFINITY;
      l[0] = l[1] = 0.f;
#pragma unroll
      for (int i = 0; i < kKS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    }
    const int pos = a.q0 + cur.t;  // the query's position; positions fit int32
    const int last = (causal && pos < n - 1) ? pos : static_cast<int>(n - 1);
    const int blk = __shfl_sync(kFull, cur.blk_lane, cur.idx);
    const int key0 = blk * CC + cur.half * kKeysPerChunk;
    const bool full = key0 + kKeysPerChunk - 1 <= last;
    const unsigned char* ks_ = ring + st * 2 * kChunkBytes;
    const unsigned char* vs_ = ks_ + kChunkBytes;

    // ---- S^T = K Q^T for the chunk's keys (16-key M tiles; two accumulators
    // each over even / odd k steps to shorten the MMA dependency chain)
    float s[kMT][4];
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
      float s2[4] = {0.f, 0.f, 0.f, 0.f};
      s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
      const int mat = lane >> 3, r = lane & 7;
      const int krow = 16 * mt + r + 8 * (mat & 1);
#pragma unroll
      for (int kk = 0; kk < kKS; ++kk) {
        uint32_t af[4];
        ldsm_x4(af, ks_ + swz128<kKeysPerChunk>(krow, 8 * (2 * kk + (mat >> 1))));
        if (kk & 1) mma_bf16(s2, af, qb[kk][0], qb[kk][1]);
        else mma_bf16(s[mt], af, qb[kk][0], qb[kk][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) s[mt][i] += s2[i];
    }
    // ---- online softmax per head (this lane: heads 2 tig, 2 tig + 1)
    float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const bool ok = full || key0 + 16 * mt + gid + 8 * rr <= last;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float x = ok ? s[mt][2 * rr + j] * a.scale : -INFINITY;
          s[mt][2 * rr + j] = x;
          bm[j] = fmaxf(bm[j], x);
        }
      }
    // Lazy rescaling: the reference maximum m of a head moves only when one
    // of its logits exceeds m by more than kLazy; o and the partial sums are
    // then rescaled. Otherwise p = exp(x - m) <= e^kLazy, which fp32 and the
    // bf16 P operand hold at full relative precision, and the chunk needs no
    // cross-lane reduction. Row sums are kept per lane and reduced at the end
    // of the row.
    if (__any_sync(kFull, bm[0] > m[0] + kLazy || bm[1] > m[1] + kLazy)) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        bm[j] = fmaxf(bm[j], __shfl_xor_sync(kFull, bm[j], 4));
        bm[j] = fmaxf(bm[j], __shfl_xor_sync(kFull, bm[j], 8));
        bm[j] = fmaxf(bm[j], __shfl_xor_sync(kFull, bm[j], 16));
        const float mn = fmaxf(m[j], bm[j]);
        const float alpha = (m[j] == -INFINITY) ? 0.f : expf(m[j] - mn);
        m[j] = mn;
        l[j] *= alpha;
#pragma unroll
        for (int md = 0; md < kKS; ++md) {
          o[md][j] *= alpha;
          o[md][2 + j] *= alpha;
        }
      }
    }
    uint32_t pb[kMT][2];
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
      float p[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = i & 1;
        p[i] = (s[mt][i] == -INFINITY) ? 0.f : expf(s[mt][i] - m[j]);
        l[j] += p[i];
      }
      pb[mt][0] = movtrans(pack_bf16(p[0], p[1]));
      pb[mt][1] = movtrans(pack_bf16(p[2], p[3]));
    }
    // ---- O^T += V^T P^T (one k step per 16 keys)
#pragma unroll
    for (int kk = 0; kk < kMT; ++kk) {
      const int mat = lane >> 3, r = lane & 7;
      const int vrow = 16 * kk + r + 8 * (mat >> 1);
#pragma unroll
      for (int md = 0; md < kKS; ++md) {
        uint32_t af[4];
        ldsm_x4_t(af, vs_ + swz128<kKeysPerChunk>(vrow, 8 * (2 * md + (mat & 1))));
        mma_bf16(o[md], af, pb[kk][0], pb[kk][1]);
      }
    }
    __syncwarp();  // this stage is refilled by the next iteration's prefetch

    if (nxt.row != cur.row) {  // last chunk of the row: write o / l and lse
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        l[j] += __shfl_xor_sync(kFull, l[j], 4);
        l[j] += __shfl_xor_sync(kFull, l[j], 8);
        l[j] += __shfl_xor_sync(kFull, l[j], 16);
      }
      const int64_t hs = nq * D;
      bf16* o0 = out + ((static_cast<int64_t>(hb) * a.H_q + hh * G) * nq + t) * D;
      float inv[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) inv[j] = l[j] > 0.f ? 1.f / l[j] : 0.f;
#pragma unroll
      for (int md = 0; md < kKS; ++md)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int d = 16 * md + gid + 8 * rr;
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (2 * tig + j < G) o0[(2 * tig + j) * hs + d] = __float2bfloat16_rn(o[md][2 * rr + j] * inv[j]);
        }
      if (lse && gid == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
          if (2 * tig + j < G) lse[(static_cast<int64_t>(hb) * a.H_q + hh * G + 2 * tig + j) * nq + t] = m[j] + logf(l[j]);
      }
    }
    cur = nxt;
    st = st + 1 == kAttnStages ? 0 : st + 1;
  }
}

int sm_count_attn() {
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

cudaError_t launch_attn_mma(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                            void* out, float* lse, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.H_kv * a.Nq;      // query rows
  const int64_t key_rows = static_cast<int64_t>(a.B) * a.H_kv * a.N;   // K and V rows
  const int64_t want = (rows + kAttnWarps - 1) / kAttnWarps;
  const unsigned grid = static_cast<unsigned>(want < sm_count_attn() ? want : sm_count_attn());
  CUtensorMap tmk, tmv;
  cudaError_t e = make_tmap_bf16_2d(&tmk, k, a.d, static_cast<uint64_t>(key_rows), kKeysPerChunk);
  if (e == cudaSuccess) e = make_tmap_bf16_2d(&tmv, v, a.d, static_cast<uint64_t>(key_rows), kKeysPerChunk);
  if (e != cudaSuccess) return e;
  unsigned long long* faults = wait_fault_counter();
  return dispatch_tdg(PISA_DTYPE_BF16, a.d, a.H_q / a.H_kv, [&](auto, auto dd, auto gg) -> cudaError_t {
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    const size_t smem = static_cast<size_t>(kAttnWarps) * kAttnStages * 2 * kKeysPerChunk * D * 2 + 1024;
    auto kern = a.C == 64 ? attn_kernel<D, 64, G> : attn_kernel<D, 32, G>;
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e2 != cudaSuccess) return e2;
    TimedLaunch tl("attn_kernel", st);
    kern<<<grid, kAttnWarps * 32, smem, st>>>(static_cast<const bf16*>(q), tmk, tmv, sel, a, static_cast<bf16*>(out),
                                              lse, faults);
    count_launch();
    return cudaGetLastError();
  });
}

}  // namespace pisa
