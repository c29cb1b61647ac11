// Fused decode step for bf16 caches (paper §Kernels, decoding): one CTA of
// four warps per (sequence, kv head) appends the new token, updates the
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
//   cores (summaries split into bf16 hi + lo), one 16-child M tile per warp.
//   Leaf candidates are scored by their exact raw-key LSE. Their key rows
//   stream through a per-warp ring of shared-memory tiles (16 keys x d each,
//   filled by cp.async ahead of use, so every warp keeps loads in flight) and
//   S^T = K Q^T is taken per tile on tensor cores. The scaled logits of every
//   candidate key go to the caller's workspace (a few tens of KB per CTA,
//   read back from L2). Top-K by warp bitonic sort; ties to the lower block
//   index.
// * Attend. The logits of the selected blocks are among those just computed
//   for the leaf level, so only V streams through the ring: O^T += V^T P^T
//   per 16-key tile under an online softmax, and the warps' partial states
//   are merged through shared memory. When the leaf level was not scored (all
//   its blocks kept, or an attend-only call) the selected blocks' keys are
//   scored first the same way.
// * Lengths. With append, the H_kv CTAs of a sequence form one thread-block
//   cluster: all of them read len[s] before the cluster barrier, after which
//   the first CTA stores len[s] + 1.
// * Caches. Dense [S, H_kv, cap, d], or paged (PAGED): leaf i of sequence s
//   in page block_table[s][i] of a pool [pages, H_kv, C, d]. Only the row
//   address differs (kv_row); the arithmetic and its order are the same.
#include <cooperative_groups.h>

#include "attn_mma.cuh"
#include "dispatch.cuh"
#include "kernels.cuh"
#include "pyramid.cuh"
#include "rowops.cuh"
#include "tma.cuh"

namespace cg = cooperative_groups;

namespace pisa {

namespace {

constexpr int kDecWarps = 4;
constexpr int kStages = 2;   // ring tiles per warp: one in use, one in flight
constexpr int kMaxCand = 32;  // leaf candidates: children of the K kept parents
static_assert(2 * kMaxK <= kMaxCand, "candidates fit one warp");
constexpr int kModeAppend = 1, kModeSelect = 2, kModeAttend = 4;

constexpr int cmax(int x, int y) { return x > y ? x : y; }

// Dynamic shared memory: the warps' tile rings during select and attend,
// reused for the append's sibling rows and leaf key rows and for the final
// merge of the warps' softmax states.
template <int D, int CC, int G>
struct DecSmem {
  static constexpr int kTile = 16 * D;  // bf16 elements per ring tile
  static constexpr int kRing = kDecWarps * kStages * kTile * 2;
  static constexpr int kState = 4 + 4 * (D / 16);  // m[2], l[2], o[D/16][4] per lane
  static constexpr int kMerge = kDecWarps * 32 * kState * 4;
  static constexpr int kSib = kMaxLevels * D * 4;
  static constexpr int kLeafOff = kSib;  // append: the leaf's key rows follow the siblings
  static constexpr int kBytes = cmax(kRing, cmax(kMerge, kLeafOff + CC * D * 2));
};

struct TileSrc {
  const bf16* p;  // row 0 of the tile
  int nvalid;     // rows that exist (the rest read as zero)
};

// Copies a 16 x D bf16 tile into shared memory by cp.async; rows at or
// beyond nvalid are zero-filled. 16-byte chunk c of row r lands at chunk
// c ^ (r & 7), so the ldmatrix reads below are free of bank conflicts.
template <int D>
__device__ inline void fill_tile(bf16* t, TileSrc src) {
  constexpr int kCh = D / 8;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = lane; i < 16 * kCh; i += 32) {
    const int r = i / kCh, c = i % kCh;
    const bool ok = r < src.nvalid;
    cp_async16(t + r * D + ((c ^ (r & 7)) << 3), src.p + (ok ? r * D + c * 8 : 0), ok ? 16 : 0);
  }
}

// Runs use(u, tile) for u = 0 .. U-1 over the tiles src(u), streamed through
// this warp's ring of kStages shared-memory tiles (kStages - 1 tiles in
// flight while one is in use).
template <int D, typename Src, typename Use>
__device__ inline void stream_tiles(bf16* ring, int U, Src src, Use use) {
  constexpr int kTile = 16 * D;
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < U) fill_tile<D>(ring + i * kTile, src(i));
    cp_async_commit();
  }
  for (int u = 0; u < U; ++u) {
    const int v = u + kStages - 1;
    if (v < U) fill_tile<D>(ring + (v % kStages) * kTile, src(v));
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncwarp();
    use(u, ring + (u % kStages) * kTile);
    __syncwarp();
  }
}

// S^T = K Q^T for the 16 key rows of a ring tile: lane (gid, tig) gets keys
// gid and gid + 8 for heads 2 tig and 2 tig + 1 (acc[2 r + j]).
template <int D>
__device__ inline void score_tile(const bf16* t, const uint32_t (&qs)[D / 16][2], float (&acc)[4]) {
  const int lane = threadIdx.x & 31, mi = lane >> 3, r = (lane & 7) + 8 * (mi & 1);
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t af[4];
    ldsm_x4(af, t + r * D + (((2 * ks + (mi >> 1)) ^ (lane & 7)) << 3));
    mma_bf16(acc, af, qs[ks][0], qs[ks][1]);
  }
}

// Stores a tile's scaled logits into a block's slot of the logit store,
// st[key][G] (key = row within the block).
template <int G>
__device__ inline void put_logits(float* st, int row0, const float (&acc)[4], float scale) {
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float* p = st + (row0 + gid + 8 * r) * G + 2 * tig;
    if constexpr (G >= 2) {
      if (2 * tig < G) *reinterpret_cast<float2*>(p) = make_float2(acc[2 * r] * scale, acc[2 * r + 1] * scale);
    } else {
      if (tig == 0) *p = acc[2 * r] * scale;
    }
  }
}

// Lane-local running log-sum-exp: (m, l) represents l * exp(m).
__device__ inline void lse_push(float& m, float& l, float x) {
  if (x == -INFINITY) return;
  if (x > m) {
    l = l * expf(m - x) + 1.f;
    m = x;
  } else {
    l += expf(x - m);
  }
}

// Asks the memory system to bring `bytes` (a multiple of 16) starting at p
// into L2, without waiting; later loads of the range then hit L2.
__device__ inline void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}

template <int D, int CC, int G, bool PAGED>
__global__ void __launch_bounds__(kDecWarps * 32, 4)
    decode_kernel(DecodeArgs a, Layout lay, int mode, const bf16* __restrict__ q_new, const bf16* __restrict__ k_new,
                  const bf16* __restrict__ v_new, bf16* __restrict__ kc, bf16* __restrict__ vc,
                  float* __restrict__ pyr, int32_t* __restrict__ len, int32_t* __restrict__ sel,
                  bf16* __restrict__ out, float* __restrict__ lse, int32_t* __restrict__ status,
                  float* lgt_ws, const int32_t* __restrict__ bt, int max_pages) {
  using LM = LeafMean<bf16, D>;
  using SM = DecSmem<D, CC, G>;
  constexpr int kKS = D / 16, kMT = CC / 16;
  extern __shared__ __align__(128) unsigned char dsm[];
  float* buf = reinterpret_cast<float*>(dsm);  // the rings' space as fp32 (siblings, merge)
  __shared__ int64_t off[kMaxLevels + 2];
  __shared__ int wcand[kDecWarps * kMaxCand];
  __shared__ float score2[2 * kMaxCand];
  __shared__ int have_lgt;
  __shared__ int blk[kMaxK], bslot[kMaxK];
  load_offsets(lay, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  bf16* ring = reinterpret_cast<bf16*>(dsm) + warp * kStages * SM::kTile;  // this warp's tiles
  const int64_t s = blockIdx.x / a.H_kv, h = blockIdx.x % a.H_kv;
  const int64_t bh = s * a.H_kv + h;
  const int C = a.C, K = a.K;
  // Element offset of key (and value) row j of this (sequence, kv head):
  // dense caches [S, H_kv, cap, D]; paged caches hold leaf j / C of the
  // sequence in page bt[s][j / C], laid out [page][H_kv][C][D].
  auto kv_row = [&](int64_t j) -> int64_t {
    if constexpr (PAGED) {
      const int64_t pg = bt[s * max_pages + j / CC];
      return ((pg * a.H_kv + h) * CC + j % CC) * D;
    } else {
      return (bh * a.cap + j) * D;
    }
  };
  const int64_t n0 = len[s];
  int64_t nn = n0;
  if (mode & kModeAppend) {
    // The appended token's leaf is averaged right after the barrier: ask for
    // its existing keys now.
    if (threadIdx.x == 0 && n0 > 0 && n0 < a.cap) {
      const int64_t lk0 = (n0 / C) * C;
      if (n0 > lk0) prefetch_l2(kc + kv_row(lk0), static_cast<uint32_t>((n0 - lk0) * D * 2));
    }
    cg::this_cluster().sync();  // every CTA of this sequence has read len[s]
    // Full: no room left, or (paged) no page for the new token's leaf.
    if (n0 >= a.cap || n0 < 0 || (PAGED && bt[s * max_pages + n0 / CC] < 0)) {
      if (h == 0 && threadIdx.x == 0) *status = PISA_ERR_CAPACITY;
    } else {
      nn = n0 + 1;
      if (h == 0 && threadIdx.x == 0) len[s] = static_cast<int32_t>(nn);
    }
  }
  if (nn <= 0 || nn > a.cap) return;
  float* P = pyr + bh * lay.R * D;
  // Logit store of this (sequence, head): [2K slots][CC keys][G heads]; null
  // when nothing is attended.
  float* lgt = lgt_ws ? lgt_ws + bh * (2 * K) * CC * G : nullptr;

  if ((mode & kModeAppend) && nn == n0 + 1) {
    const int64_t n = n0;  // position of the new token
    const int64_t leaf = n / C;
    const int L = num_levels(nn, C);
    // The leaf's existing key rows are staged in shared memory by cp.async
    // while the path's left siblings are read, so both cost one memory round
    // trip; the new token's row is taken from k_new.
    bf16* lrows = reinterpret_cast<bf16*>(dsm + SM::kLeafOff);  // [C][D]
    const int64_t lo = leaf * C;
    const int nold = static_cast<int>(n - lo);
    for (int i = threadIdx.x; i < nold * (D / 8); i += blockDim.x) {
      const int r = i / (D / 8), c8 = i % (D / 8);
      cp_async16(lrows + r * D + c8 * 8, kc + kv_row(lo + r) + c8 * 8, 16);
    }
    cp_async_commit();
    if (warp == 0) {
      bf16* kr = kc + kv_row(n);
      bf16* vr = vc + kv_row(n);
      for (int e = lane; e < D / 2; e += 32) {
        const uint32_t kw = reinterpret_cast<const uint32_t*>(k_new + bh * D)[e];
        reinterpret_cast<uint32_t*>(kr)[e] = kw;
        reinterpret_cast<uint32_t*>(lrows + nold * D)[e] = kw;
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
    cp_async_wait<0>();
    __threadfence_block();
    __syncthreads();
    if (warp == 0) {
      float mean[LM::kVec];
      leaf_mean_warp<bf16, D>(lrows, 0, nold + 1, mean);
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

  // Query heads of the group as MMA B fragments (zero beyond G): qs in the
  // plain k order (for ldmatrix A operands), qb with four contiguous d per
  // lane (for the router's fp32 summary rows).
  uint32_t qs[kKS][2];
  {
    const bf16* qp = q_new + (s * a.H_q + h * G + (gid < G ? gid : 0)) * D + 2 * tig;
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
      qs[ks][0] = gid < G ? *reinterpret_cast<const uint32_t*>(qp + 16 * ks) : 0u;
      qs[ks][1] = gid < G ? *reinterpret_cast<const uint32_t*>(qp + 16 * ks + 8) : 0u;
    }
  }
  if (threadIdx.x == 0) have_lgt = 0;

  if (mode & kModeSelect) {
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
    // Highest level with more than K blocks (all blocks are usable by the
    // last token); every level above it keeps all its blocks unscored.
    int l = num_levels(nn, C);
    while (l >= 1 && level_size(nn, C, l) <= K) --l;
    if (l < 1) {
      const int tx = static_cast<int>(threadIdx.x);
      if (tx < K) blk[tx] = tx < level_size(nn, C, 1) ? tx : -1;
    } else {
      // Every warp holds the candidate list (lane i: candidate i) and takes
      // the same top-K decisions from the shared scores, so a level costs one
      // CTA barrier; scored levels alternate between two score buffers, so a
      // warp that runs ahead never overwrites scores another warp still reads.
      int c = lane < level_size(nn, C, l) ? lane : -1;
      int nc = static_cast<int>(level_size(nn, C, l));
      int* wc = wcand + warp * kMaxCand;  // this warp's copy, for indexed reads
      for (int p = 0;; --l) {
        float* sc = score2 + p * kMaxCand;
        const bool scored = nc > K;
        if (scored) {
          if (l >= 2) {
            // Warp m scores candidates 8m .. 8m+7 by their two children.
            const int m = warp;
            const int cm = __shfl_sync(kFull, c, (8 * m + gid) & 31);
            if (8 * m < nc) {
              const bool have = 8 * m + gid < nc;
              const int64_t cc = have ? cm : 0;
              const bool has1 = have && 2 * cc + 1 < level_size(nn, C, l - 1);
              const float* p0 = P + (off[l - 1] + 2 * cc) * D + 4 * tig;
              const float* p1 = P + (off[l - 1] + (has1 ? 2 * cc + 1 : 2 * cc)) * D + 4 * tig;
              float acc[4] = {0.f, 0.f, 0.f, 0.f};
              // Both children's rows are loaded before any use, so the level
              // costs one memory round trip.
              float4 x0[kKS], x1[kKS];
#pragma unroll
              for (int ks = 0; ks < kKS; ++ks) {
                x0[ks] = *reinterpret_cast<const float4*>(p0 + 16 * ks);
                x1[ks] = *reinterpret_cast<const float4*>(p1 + 16 * ks);
              }
#pragma unroll
              for (int ks = 0; ks < kKS; ++ks) {
                uint32_t hi[4], lo[4];
                a_split(x0[ks], x1[ks], hi, lo);
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
              if (tig == 0 && have) sc[8 * m + gid] = u;
            }
          } else {
            // Leaf candidates x = warp, warp + 4, ...: their key tiles stream
            // through the ring; each tile's logits go to the store and into a
            // lane-local running LSE per head, reduced when the leaf ends.
            wc[lane] = c;
            __syncwarp();
            const int nxw = nc > warp ? (nc - warp + kDecWarps - 1) / kDecWarps : 0;
            float lm[2] = {-INFINITY, -INFINITY}, ll[2] = {0.f, 0.f};
            stream_tiles<D>(
                ring, nxw * kMT,
                [&](int u) -> TileSrc {
                  const int64_t k0 = static_cast<int64_t>(wc[warp + kDecWarps * (u / kMT)]) * CC + 16 * (u % kMT);
                  const int64_t nv = nn - k0;
                  return nv > 0 ? TileSrc{kc + kv_row(k0), nv < 16 ? static_cast<int>(nv) : 16} : TileSrc{kc, 0};
                },
                [&](int u, const bf16* t) {
                  const int x = warp + kDecWarps * (u / kMT), mt = u % kMT;
                  const int64_t k0 = static_cast<int64_t>(wc[x]) * CC + 16 * mt;
                  float acc[4];
                  score_tile<D>(t, qs, acc);
                  if (lgt) put_logits<G>(lgt + x * CC * G, 16 * mt, acc, a.scale);
#pragma unroll
                  for (int r = 0; r < 2; ++r)
                    if (k0 + gid + 8 * r < nn) {
                      lse_push(lm[0], ll[0], acc[2 * r] * a.scale);
                      lse_push(lm[1], ll[1], acc[2 * r + 1] * a.scale);
                    }
                  if (mt == kMT - 1) {
                    float u2 = 0.f;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                      float mx = lm[j];
                      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
                      float sm = lm[j] == -INFINITY ? 0.f : ll[j] * expf(lm[j] - mx);
                      sm += __shfl_xor_sync(kFull, sm, 4);
                      sm += __shfl_xor_sync(kFull, sm, 8);
                      sm += __shfl_xor_sync(kFull, sm, 16);
                      if (2 * tig + j < G) u2 += mx + logf(sm);
                      lm[j] = -INFINITY;
                      ll[j] = 0.f;
                    }
                    u2 += __shfl_xor_sync(kFull, u2, 1);
                    u2 += __shfl_xor_sync(kFull, u2, 2);
                    if (lane == 0) sc[x] = u2;
                  }
                });
          }
          __syncthreads();
        }
        // Kept blocks of this level: the K best when scored, else all.
        int idx = lane < nc ? c : INT_MAX;
        int nk = nc;
        if (scored) {
          float v = lane < nc ? sc[lane] : -INFINITY;
          warp_sort_desc(v, idx);
          nk = K;
          p ^= 1;  // the next scored level writes the other buffer
        }
        if (l == 1) {
          if (warp == 0) {
            int kept = lane < nk ? idx : INT_MAX;
            warp_sort_asc(kept);
            if (lane < K) {
              blk[lane] = kept == INT_MAX ? -1 : kept;
              // Slot of the kept leaf in the logit store.
              int sl = 0;
              for (int x = 0; x < nc; ++x)
                if (wc[x] == kept) sl = x;
              bslot[lane] = sl;
            }
            if (lane == 0) have_lgt = scored ? 1 : 0;
          }
          break;
        }
        // Children of the kept blocks that exist, compacted to the front.
        const int parent = __shfl_sync(kFull, idx, lane >> 1);
        const int64_t child = 2 * static_cast<int64_t>(parent) + (lane & 1);
        c = static_cast<int>(child);
        nc = warp_compact(c, (lane >> 1) < nk && child < level_size(nn, C, l - 1), wc);
      }
    }
    __syncthreads();
    if (sel && threadIdx.x < K) sel[bh * K + threadIdx.x] = blk[threadIdx.x];
  } else if (warp == 0) {
    // Selections passed in: their valid entries, in order, as a prefix.
    int b = lane < K ? sel[bh * K + lane] : -1;
    warp_compact(b, b >= 0, wcand);
    if (lane < K) blk[lane] = b;
  }
  __syncthreads();

  if (mode & kModeAttend) {
    // Selected blocks: an ascending prefix of blk; warp w takes x = w, w + 4, ...
    int nsel = 0;
    for (int x = 0; x < K; ++x) nsel += blk[x] >= 0;
    const int nbw = nsel > warp ? (nsel - warp + kDecWarps - 1) / kDecWarps : 0;
    if (!have_lgt) {
      // Logits of the selected blocks' keys, into slots x (warp-private).
      stream_tiles<D>(
          ring, nbw * kMT,
          [&](int u) -> TileSrc {
            const int64_t k0 = static_cast<int64_t>(blk[warp + kDecWarps * (u / kMT)]) * CC + 16 * (u % kMT);
            const int64_t nv = nn - k0;
            return nv > 0 ? TileSrc{kc + kv_row(k0), nv < 16 ? static_cast<int>(nv) : 16} : TileSrc{kc, 0};
          },
          [&](int u, const bf16* t) {
            const int x = warp + kDecWarps * (u / kMT);
            float acc[4];
            score_tile<D>(t, qs, acc);
            put_logits<G>(lgt + x * CC * G, 16 * (u % kMT), acc, a.scale);
          });
    }
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[kKS][4];
#pragma unroll
    for (int i = 0; i < kKS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    stream_tiles<D>(
        ring, nbw * kMT,
        [&](int u) -> TileSrc {
          const int64_t k0 = static_cast<int64_t>(blk[warp + kDecWarps * (u / kMT)]) * CC + 16 * (u % kMT);
          const int64_t nv = nn - k0;
          return nv > 0 ? TileSrc{vc + kv_row(k0), nv < 16 ? static_cast<int>(nv) : 16} : TileSrc{vc, 0};
        },
        [&](int u, const bf16* t) {
          const int x = warp + kDecWarps * (u / kMT), kk = u % kMT;
          const int64_t k0 = static_cast<int64_t>(blk[x]) * CC + 16 * kk;
          const int sl = have_lgt ? bslot[x] : x;
          const float* lp = lgt + (sl * CC + 16 * kk) * G;
          float sv[4];
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int j = 0; j < 2; ++j)
              sv[2 * r + j] = (k0 + gid + 8 * r < nn && 2 * tig + j < G) ? lp[(gid + 8 * r) * G + 2 * tig + j]
                                                                          : -INFINITY;
          float mn[2], alpha[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            float bm = fmaxf(sv[j], sv[2 + j]);
            bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 4));
            bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 8));
            bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 16));
            mn[j] = fmaxf(m[j], bm);
            alpha[j] = m[j] == -INFINITY ? 0.f : expf(m[j] - mn[j]);
            m[j] = mn[j];
          }
          float p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) p[i] = sv[i] == -INFINITY ? 0.f : expf(sv[i] - mn[i & 1]);
#pragma unroll
          for (int j = 0; j < 2; ++j) l[j] = l[j] * alpha[j] + p[j] + p[2 + j];  // lane-local partial sums
#pragma unroll
          for (int md = 0; md < kKS; ++md) {
            o[md][0] *= alpha[0];
            o[md][1] *= alpha[1];
            o[md][2] *= alpha[0];
            o[md][3] *= alpha[1];
          }
          // P^T (keys x heads) as B fragments by transposition; V^T tiles by
          // transposing ldmatrix reads of the V rows.
          const uint32_t pb0 = movtrans(pack_bf16(p[0], p[1])), pb1 = movtrans(pack_bf16(p[2], p[3]));
          const int mi = lane >> 3, rv = (lane & 7) + 8 * (mi >> 1);
#pragma unroll
          for (int md = 0; md < kKS; ++md) {
            uint32_t af[4];
            ldsm_x4_t(af, t + rv * D + (((2 * md + (mi & 1)) ^ (lane & 7)) << 3));
            mma_bf16(o[md], af, pb0, pb1);
          }
        });
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      l[j] += __shfl_xor_sync(kFull, l[j], 4);
      l[j] += __shfl_xor_sync(kFull, l[j], 8);
      l[j] += __shfl_xor_sync(kFull, l[j], 16);
    }
    __syncthreads();  // every warp is done with its ring: the space becomes the merge area
    float* st = buf + (warp * 32 + lane) * SM::kState;
    st[0] = m[0];
    st[1] = m[1];
    st[2] = l[0];
    st[3] = l[1];
#pragma unroll
    for (int i = 0; i < kKS; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) st[4 + 4 * i + j] = o[i][j];
    __syncthreads();
    if (warp == 0) {
      for (int w = 1; w < kDecWarps; ++w) {
        const float* o2 = buf + (w * 32 + lane) * SM::kState;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float m2 = o2[j], l2 = o2[2 + j];
          const float mx = fmaxf(m[j], m2);
          const float a1 = m[j] == -INFINITY ? 0.f : expf(m[j] - mx);
          const float a2 = m2 == -INFINITY ? 0.f : expf(m2 - mx);
          l[j] = l[j] * a1 + l2 * a2;
#pragma unroll
          for (int md = 0; md < kKS; ++md) {
            o[md][j] = o[md][j] * a1 + o2[4 + 4 * md + j] * a2;
            o[md][2 + j] = o[md][2 + j] * a1 + o2[4 + 4 * md + 2 + j] * a2;
          }
          m[j] = mx;
        }
      }
      // O^T rows are d = 16 md + gid (+8), columns heads 2 tig + j.
      bf16* ob = out + (s * a.H_q + h * G) * D;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int hd = 2 * tig + j;
        if (hd >= G) continue;
        const float inv = l[j] > 0.f ? 1.f / l[j] : 0.f;
#pragma unroll
        for (int md = 0; md < kKS; ++md)
#pragma unroll
          for (int r = 0; r < 2; ++r) store_out(ob + hd * D + 16 * md + gid + 8 * r, o[md][2 * r + j] * inv);
        if (lse && gid == 0) lse[s * a.H_q + h * G + hd] = m[j] + logf(l[j]);
      }
    }
  }
}

}  // namespace

bool decode_fused_supported(const DecodeArgs& a) {
  return a.dtype == PISA_DTYPE_BF16 && a.H_kv <= 8 && a.H_q / a.H_kv <= 8;
}

int64_t decode_logit_floats(const DecodeArgs& a) {
  return static_cast<int64_t>(a.S) * a.H_kv * (2 * a.K) * a.C * (a.H_q / a.H_kv);
}

cudaError_t launch_decode_fused(const DecodeArgs& a, const Layout& lay, int mode, const void* q_new,
                                const void* k_new, const void* v_new, void* k_cache, void* v_cache, float* pyr,
                                int32_t* len, int32_t* sel, void* out, float* lse, int32_t* status, float* lgt_ws,
                                cudaStream_t st, const int32_t* block_table, int max_pages) {
  return dispatch_tdg(PISA_DTYPE_BF16, a.d, a.H_q / a.H_kv, [&](auto, auto dd, auto gg) -> cudaError_t {
    constexpr int D = decltype(dd)::value, G = decltype(gg)::value;
    auto kern = block_table ? (a.C == 64 ? decode_kernel<D, 64, G, true> : decode_kernel<D, 32, G, true>)
                            : (a.C == 64 ? decode_kernel<D, 64, G, false> : decode_kernel<D, 32, G, false>);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.S * a.H_kv));
    cfg.blockDim = dim3(kDecWarps * 32);
    const int smem = DecSmem<D, 64, G>::kBytes;  // covers both block sizes
    cudaError_t e0 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e0 != cudaSuccess) return e0;
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (mode & kModeAppend) ? static_cast<unsigned>(a.H_kv) : 1u;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TimedLaunch tl("decode_kernel", st);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, lay, mode, static_cast<const bf16*>(q_new),
                                       static_cast<const bf16*>(k_new), static_cast<const bf16*>(v_new),
                                       static_cast<bf16*>(k_cache), static_cast<bf16*>(v_cache), pyr, len, sel,
                                       static_cast<bf16*>(out), lse, status, lgt_ws, block_table, max_pages);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  });
}

}  // namespace pisa
