// Fused decode step for bf16 caches (paper §Kernels, decoding): one CTA of
// eight warps per (sequence, kv head) appends the new token, updates the
// cached mean pyramid along the new leaf's ancestor path, selects K leaf
// blocks root-to-leaf (scoring raw keys at the leaf level) and attends the
// new query over them, all in one launch with the selection kept on chip.
//
// * Append. The new token is the last one, so its ancestors form the
//   rightmost path of the tree: a path node is either a lone left child or
//   the right child of an unchanged left sibling. The siblings are read
//   first (by all warps, in parallel); the path is then a short chain of
//   register updates, each node the mean of its existing children (same
//   arithmetic and order as the batch build).
// * Select. Inner levels score the children of <= 2K candidates on tensor
//   cores (summaries split into bf16 hi + lo), one 16-child M tile per warp;
//   leaf candidates are scored by their exact raw-key LSE, one leaf per warp
//   at a time. Top-K by warp bitonic sort; ties to the lower block index.
// * Attend. The selected blocks are spread over the warps (MmaAttend) and
//   the partial softmax states are merged through shared memory.
// * Lengths. With append, the H_kv CTAs of a sequence form one thread-block
//   cluster: all of them read len[s] before the cluster barrier, after which
//   the first CTA stores len[s] + 1.
#include <cooperative_groups.h>

#include "attn_mma.cuh"
#include "dispatch.cuh"
#include "kernels.cuh"
#include "pyramid.cuh"
#include "rowops.cuh"

namespace cg = cooperative_groups;

namespace pisa {

namespace {

constexpr int kDecWarps = 8;
constexpr int kModeAppend = 1, kModeSelect = 2, kModeAttend = 4;

// Asks the memory system to bring `bytes` (a multiple of 16) starting at p
// into L2, without waiting; later loads of the range then hit L2.
__device__ inline void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}

// Raw-key LSE of one leaf block summed over the G heads, by one warp
// (S^T = K Q^T on tensor cores; keys at or beyond n are excluded).
template <int D, int CC, int G>
__device__ inline float leaf_lse(const bf16* __restrict__ kh, int64_t key0, int64_t n, const uint32_t (&qb)[D / 16][2],
                                 float scale) {
  constexpr int kKS = D / 16, kMT = CC / 16;
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int64_t last = n - 1;
  float s[kMT][4];
#pragma unroll
  for (int mt = 0; mt < kMT; ++mt) {
    const int64_t k0 = key0 + 16 * mt + gid;
    const bf16* pa = kh + (k0 <= last ? k0 : last) * D + 4 * tig;
    const bf16* pb = kh + (k0 + 8 <= last ? k0 + 8 : last) * D + 4 * tig;
    uint2 ua[kKS], ub[kKS];
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
      ua[ks] = __ldg(reinterpret_cast<const uint2*>(pa + 16 * ks));
      ub[ks] = __ldg(reinterpret_cast<const uint2*>(pb + 16 * ks));
    }
    s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
      const uint32_t a[4] = {ua[ks].x, ub[ks].x, ua[ks].y, ub[ks].y};
      mma_bf16(s[mt], a, qb[ks][0], qb[ks][1]);
    }
  }
  float u = 0.f;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float mx = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
      for (int r = 0; r < 2; ++r)
        if (key0 + 16 * mt + gid + 8 * r <= last) mx = fmaxf(mx, s[mt][2 * r + j]);
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
    float sum = 0.f;
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
      for (int r = 0; r < 2; ++r)
        if (key0 + 16 * mt + gid + 8 * r <= last) sum += expf((s[mt][2 * r + j] - mx) * scale);
    sum += __shfl_xor_sync(kFull, sum, 4);
    sum += __shfl_xor_sync(kFull, sum, 8);
    sum += __shfl_xor_sync(kFull, sum, 16);
    if (2 * tig + j < G) u += mx * scale + logf(sum);
  }
  u += __shfl_xor_sync(kFull, u, 1);
  u += __shfl_xor_sync(kFull, u, 2);
  return u;
}

template <int D, int CC, int G>
__global__ void __launch_bounds__(kDecWarps * 32, 2)
    decode_kernel(DecodeArgs a, Layout lay, int mode, const bf16* __restrict__ q_new, const bf16* __restrict__ k_new,
                  const bf16* __restrict__ v_new, bf16* __restrict__ kc, bf16* __restrict__ vc,
                  float* __restrict__ pyr, int32_t* __restrict__ len, int32_t* __restrict__ sel,
                  bf16* __restrict__ out, float* __restrict__ lse, int32_t* __restrict__ status) {
  using LM = LeafMean<bf16, D>;
  constexpr int kKS = D / 16;
  constexpr int kState = 4 + 4 * kKS;  // m[2], l[2], o[kKS][4] per lane
  __shared__ int64_t off[kMaxLevels + 2];
  __shared__ __align__(16) float buf[kDecWarps * 32 * kState > kMaxLevels * D ? kDecWarps * 32 * kState
                                                                               : kMaxLevels * D];
  __shared__ int cand[32];
  __shared__ float score[32];
  __shared__ int ncand_sh;
  __shared__ int blk[kMaxK];
  load_offsets(lay, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t s = blockIdx.x / a.H_kv, h = blockIdx.x % a.H_kv;
  const int64_t bh = s * a.H_kv + h;
  const int C = a.C, K = a.K;
  const int64_t n0 = len[s];
  int64_t nn = n0;
  if (mode & kModeAppend) {
    cg::this_cluster().sync();  // every CTA of this sequence has read len[s]
    if (n0 >= a.cap || n0 < 0) {
      if (h == 0 && threadIdx.x == 0) *status = PISA_ERR_CAPACITY;
    } else {
      nn = n0 + 1;
      if (h == 0 && threadIdx.x == 0) len[s] = static_cast<int32_t>(nn);
    }
  }
  if (nn <= 0 || nn > a.cap) return;
  const bf16* kh = kc + bh * a.cap * D;
  const bf16* vh = vc + bh * a.cap * D;
  float* P = pyr + bh * lay.R * D;

  if ((mode & kModeAppend) && nn == n0 + 1) {
    const int64_t n = n0;  // position of the new token
    const int64_t leaf = n / C;
    const int L = num_levels(nn, C);
    if (warp == 0) {
      bf16* kr = kc + (bh * a.cap + n) * D;
      bf16* vr = vc + (bh * a.cap + n) * D;
      for (int e = lane; e < D / 2; e += 32) {
        reinterpret_cast<uint32_t*>(kr)[e] = reinterpret_cast<const uint32_t*>(k_new + bh * D)[e];
        reinterpret_cast<uint32_t*>(vr)[e] = reinterpret_cast<const uint32_t*>(v_new + bh * D)[e];
      }
    }
    // Left siblings of the path (unchanged rows), one per level where the
    // path node is a right child.
    for (int x = threadIdx.x; x < (L - 1) * D; x += blockDim.x) {
      const int l = 2 + x / D, e = x % D;
      const int64_t c = leaf >> (l - 2);
      if (c & 1) buf[(l - 2) * D + e] = P[(off[l - 1] + c - 1) * D + e];
    }
    __threadfence_block();
    __syncthreads();
    if (warp == 0) {
      float mean[LM::kVec];
      leaf_mean_warp<bf16, D>(kh, leaf * C, nn, mean);
      LM::store(mean, nullptr, P + (off[1] + leaf) * D, lane);
      for (int l = 2; l <= L; ++l) {
        const int64_t c = leaf >> (l - 2);
        if ((c & 1) && lane < LM::kLpr) {
#pragma unroll
          for (int e = 0; e < LM::kVec; ++e) mean[e] = mean2(buf[(l - 2) * D + lane * LM::kVec + e], mean[e]);
        }
        LM::store(mean, nullptr, P + (off[l] + (c >> 1)) * D, lane);
      }
    }
    __threadfence_block();
    __syncthreads();
  }

  if (!(mode & (kModeSelect | kModeAttend))) return;  // append only: q_new and sel are not given

  // Query heads of the group as MMA B fragments (zero beyond G).
  uint32_t qb[kKS][2];
  {
    const bf16* qp = q_new + (s * a.H_q + h * G + (gid < G ? gid : 0)) * D + 4 * tig;
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
      uint2 u = make_uint2(0u, 0u);
      if (gid < G) u = *reinterpret_cast<const uint2*>(qp + 16 * ks);
      qb[ks][0] = u.x;
      qb[ks][1] = u.y;
    }
  }

  if (mode & kModeSelect) {
    // Highest level with more than K blocks (all blocks are usable by the
    // last token); every level above it keeps all its blocks unscored.
    int l = num_levels(nn, C);
    while (l >= 1 && level_size(nn, C, l) <= K) --l;
    if (l < 1) {
      const int tx = static_cast<int>(threadIdx.x);
      if (tx < K) blk[tx] = tx < level_size(nn, C, 1) ? tx : -1;
    } else {
      const int tx = static_cast<int>(threadIdx.x);
      if (tx < 32) cand[tx] = tx < level_size(nn, C, l) ? tx : -1;
      __syncthreads();
      for (;; --l) {
        // Existing candidates, compacted (warp 0), then scored if more than K.
        if (warp == 0) {
          int c = cand[lane];
          const int nc = warp_compact(c, c >= 0 && c < level_size(nn, C, l), reinterpret_cast<int*>(score));
          cand[lane] = c;
          if (lane == 0) ncand_sh = nc;
        }
        __syncthreads();
        const int nc = ncand_sh;
        const bool scored = nc > K;
        if (scored) {
          if (l >= 2) {
            const int m = warp;  // M tile: candidates 8m .. 8m+7
            if (m < 4 && 8 * m < nc) {
              const bool have = 8 * m + gid < nc;
              const int64_t c = have ? cand[8 * m + gid] : 0;
              const bool has1 = have && 2 * c + 1 < level_size(nn, C, l - 1);
              const float* p0 = P + (off[l - 1] + 2 * c) * D + 4 * tig;
              const float* p1 = P + (off[l - 1] + (has1 ? 2 * c + 1 : 2 * c)) * D + 4 * tig;
              float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int ks = 0; ks < kKS; ++ks) {
                const float4 x0 = *reinterpret_cast<const float4*>(p0 + 16 * ks);
                const float4 x1 = *reinterpret_cast<const float4*>(p1 + 16 * ks);
                uint32_t hi[4], lo[4];
                a_split(x0, x1, hi, lo);
                mma_bf16(acc, hi, qb[ks][0], qb[ks][1]);
                mma_bf16(acc, lo, qb[ks][0], qb[ks][1]);
              }
              float u = 0.f;
#pragma unroll
              for (int j = 0; j < 2; ++j)
                if (2 * tig + j < G) {
                  const float s0 = a.scale * acc[j];
                  u += has1 ? lse2(s0, a.scale * acc[2 + j]) : s0;
                }
              u += __shfl_xor_sync(kFull, u, 1);
              u += __shfl_xor_sync(kFull, u, 2);
              if (tig == 0 && have) score[8 * m + gid] = u;
            }
          } else {
            // All candidate leaves' key tiles are requested into L2 at once, so
            // their DRAM fetches overlap instead of following one another.
            if (threadIdx.x < nc) {
              const int64_t k0 = static_cast<int64_t>(cand[threadIdx.x]) * CC;
              const int64_t nk = (k0 + CC <= nn ? CC : nn - k0);
              prefetch_l2(kh + k0 * D, static_cast<uint32_t>(nk * D * 2));
            }
            for (int x = warp; x < nc; x += kDecWarps) {
              const float u = leaf_lse<D, CC, G>(kh, static_cast<int64_t>(cand[x]) * CC, nn, qb, a.scale);
              if (lane == 0) score[x] = u;
            }
          }
        }
        __syncthreads();
        if (warp == 0) {
          int idx = lane < nc ? cand[lane] : INT_MAX;
          int nk = nc;
          if (scored) {
            float sc = lane < nc ? score[lane] : -INFINITY;
            warp_sort_desc(sc, idx);
            nk = K;
          }
          if (l == 1) {
            int kept = lane < nk ? idx : INT_MAX;
            warp_sort_asc(kept);
            if (lane < K) blk[lane] = kept == INT_MAX ? -1 : kept;
          } else {
            const int parent = __shfl_sync(kFull, idx, lane >> 1);
            cand[lane] = (lane >> 1) < nk ? 2 * parent + (lane & 1) : -1;
          }
        }
        __syncthreads();
        if (l == 1) break;
      }
    }
    __syncthreads();
    if (sel && threadIdx.x < K) sel[bh * K + threadIdx.x] = blk[threadIdx.x];
  } else if ((mode & kModeAttend) && threadIdx.x < K) {
    blk[threadIdx.x] = sel[bh * K + threadIdx.x];
  }
  __syncthreads();

  if (mode & kModeAttend) {
    // The selected blocks' K and V rows are requested into L2 together.
    if (threadIdx.x < 2 * K) {
      const int bsel = blk[threadIdx.x >> 1];
      if (bsel >= 0) {
        const int64_t k0 = static_cast<int64_t>(bsel) * CC;
        const int64_t nk = (k0 + CC <= nn ? CC : nn - k0);
        prefetch_l2(((threadIdx.x & 1) ? vh : kh) + k0 * D, static_cast<uint32_t>(nk * D * 2));
      }
    }
    MmaAttend<D, CC, G> at;
    at.m[0] = at.m[1] = -INFINITY;
    at.l[0] = at.l[1] = 0.f;
#pragma unroll
    for (int i = 0; i < kKS; ++i) {
      at.o[i][0] = at.o[i][1] = at.o[i][2] = at.o[i][3] = 0.f;
      at.qb[i][0] = qb[i][0];
      at.qb[i][1] = qb[i][1];
    }
    for (int x = warp; x < K; x += kDecWarps) {
      const int b = blk[x];
      if (b >= 0) at.block(kh, vh, static_cast<int64_t>(b) * CC, nn, nn - 1, true, a.scale);
    }
    float* st = buf + (warp * 32 + lane) * kState;
    st[0] = at.m[0];
    st[1] = at.m[1];
    st[2] = at.l[0];
    st[3] = at.l[1];
#pragma unroll
    for (int i = 0; i < kKS; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) st[4 + 4 * i + j] = at.o[i][j];
    __syncthreads();
    if (warp == 0) {
      for (int w = 1; w < kDecWarps; ++w) {
        const float* o2 = buf + (w * 32 + lane) * kState;
        float m2[2] = {o2[0], o2[1]}, l2[2] = {o2[2], o2[3]};
        float oo[kKS][4];
#pragma unroll
        for (int i = 0; i < kKS; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) oo[i][j] = o2[4 + 4 * i + j];
        at.merge(m2, l2, oo);
      }
      at.store(out + (s * a.H_q + h * G) * D, D, lse ? lse + s * a.H_q + h * G : nullptr, 1);
    }
  }
}

}  // namespace

bool decode_fused_supported(const DecodeArgs& a) {
  return a.dtype == PISA_DTYPE_BF16 && a.H_kv <= 8 && a.H_q / a.H_kv <= 8;
}

cudaError_t launch_decode_fused(const DecodeArgs& a, const Layout& lay, int mode, const void* q_new,
                                const void* k_new, const void* v_new, void* k_cache, void* v_cache, float* pyr,
                                int32_t* len, int32_t* sel, void* out, float* lse, int32_t* status, cudaStream_t st) {
  return dispatch_tdg(PISA_DTYPE_BF16, a.d, a.H_q / a.H_kv, [&](auto, auto dd, auto gg) -> cudaError_t {
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    auto kern = a.C == 64 ? decode_kernel<D, 64, G> : decode_kernel<D, 32, G>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.S * a.H_kv));
    cfg.blockDim = dim3(kDecWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (mode & kModeAppend) ? static_cast<unsigned>(a.H_kv) : 1u;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, lay, mode, static_cast<const bf16*>(q_new),
                                       static_cast<const bf16*>(k_new), static_cast<const bf16*>(v_new),
                                       static_cast<bf16*>(k_cache), static_cast<bf16*>(v_cache), pyr, len, sel,
                                       static_cast<bf16*>(out), lse, status);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  });
}

}  // namespace pisa
