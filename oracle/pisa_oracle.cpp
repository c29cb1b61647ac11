// Plain, slow fp64 CPU oracle for the PISA hot path.
//
// TEST INFRASTRUCTURE ONLY. Only tests/, the smoke check and the benchmark's
// CPU-baseline leg may load this library. The product path (the CUDA library)
// never calls it and shares no code, header, table or helper with it.
//
// Every function below restates a step of "Block Sparse Attention with
// Log-Linear Complexity" as given on its hyper.ai page (the translated paper
// body). Citations name that page's sections:
//   §BSA      = "Block-sparse attention" (the attention equation for o_t)
//   §Pyramid  = "Pyramid key-block hierarchy" (level sizes, Concat, mean pooling)
//   §TopK     = "Coarse-to-fine Top-K selection" (candidate sets, LSE score)
//   §Kernels  = "Kernel implementation" (GQA score sum, decode cache update)
// Readings where the page is silent (causality, ragged blocks, tie order,
// output order) are stated at the point of use.
//
// Arithmetic is fp64 throughout. Inputs arrive in their storage format
// (fp32, or bf16 as raw 16-bit patterns) and are widened exactly to double.
// Indices are 0-based: the page's root block "1" is block 0 here.
//
// Build: g++ -O2 -fopenmp -shared -fPIC -std=c++17 pisa_oracle.cpp

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

namespace {

// Problem description shared by every oracle entry point. All integers are
// int64 so that the ctypes mirror has no padding surprises.
struct Cfg {
  int64_t B, N, H_q, H_kv, d, C, K;
  int64_t causal;  // 1: a query at position t may only use keys <= t
  int64_t dtype;   // 0: fp32 storage, 1: bf16 storage (raw 16-bit patterns)
  int64_t Nq;      // number of query positions held in q / out
  int64_t q_t0;    // position of the first held query row
  double scale;    // logit scale; <= 0 selects 1/sqrt(d) (§BSA)
};

// Widen one stored element to double. bf16 is the upper half of an IEEE
// binary32, so shifting its 16 bits up gives the exact float value.
double elem(const void* p, int64_t idx, int64_t dtype) {
  if (dtype == 0) return static_cast<double>(static_cast<const float*>(p)[idx]);
  uint32_t bits = static_cast<uint32_t>(static_cast<const uint16_t*>(p)[idx]) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return static_cast<double>(f);
}

double cfg_scale(const Cfg& c) {
  return c.scale > 0 ? c.scale : 1.0 / std::sqrt(static_cast<double>(c.d));
}

// §Pyramid: M_0 = N raw keys; the first merge uses g_0 = C (leaf blocks of C
// keys), every later merge g = 2, M_{l+1} = ceil(M_l / g_l). The hierarchy
// stops at the single root block. Returns M[0..L].
std::vector<int64_t> level_sizes(int64_t N, int64_t C) {
  std::vector<int64_t> M;
  M.push_back(N);
  if (N <= 0) return M;
  M.push_back((N + C - 1) / C);
  while (M.back() > 1) M.push_back((M.back() + 1) / 2);
  return M;
}

// Row offset of level l (1..L) inside one head's pyramid: levels are stored
// finest first, level 1 (leaves) at offset 0.
std::vector<int64_t> level_offsets(const std::vector<int64_t>& M) {
  std::vector<int64_t> off(M.size() + 1, 0);
  for (size_t l = 1; l < M.size(); ++l) off[l + 1] = off[l] + M[l];
  return off;  // off[1] = 0, off[L + 1] = R
}

// Number of keys spanned by a nominal block of level l >= 1: C * 2^(l-1).
int64_t span(int64_t C, int64_t l) { return C << (l - 1); }

// Causal validity reading (the page does not state causality): a block of
// level l >= 1 is usable by the query at position t iff its first key is
// <= t; a raw key j (level 0) iff j <= t. Non-causal: every existing block.
bool valid_block(const Cfg& c, const std::vector<int64_t>& M, int64_t l, int64_t i, int64_t t) {
  if (i < 0 || i >= M[l]) return false;
  if (!c.causal) return true;
  int64_t first = (l == 0) ? i : i * span(c.C, l);
  return first <= t;
}

// Children of block i at level l >= 1, as indices at level l-1 (§Pyramid:
// K_i^{(l)} is the Concat of its children). Leaves (l = 1) have the raw keys
// [iC, min(iC + C, N)) as children; higher levels the pair {2i, 2i+1} cut to
// the blocks that exist. Every existing child is returned; validity is a
// separate test.
std::vector<int64_t> children(const Cfg& c, const std::vector<int64_t>& M, int64_t l, int64_t i) {
  std::vector<int64_t> ch;
  if (l == 1) {
    for (int64_t j = i * c.C; j < std::min((i + 1) * c.C, c.N); ++j) ch.push_back(j);
  } else {
    for (int64_t r = 2 * i; r < std::min(2 * i + 2, M[l - 1]); ++r) ch.push_back(r);
  }
  return ch;
}

// log(sum(exp(x))) evaluated around the maximum so that it cannot overflow.
double logsumexp(const std::vector<double>& x) {
  double m = -std::numeric_limits<double>::infinity();
  for (double v : x) m = std::max(m, v);
  if (!std::isfinite(m)) return m;
  double s = 0;
  for (double v : x) s += std::exp(v - m);
  return m + std::log(s);
}

// Pointer arithmetic for the [B, H, rows, d] tensors.
int64_t q_index(const Cfg& c, int64_t b, int64_t hq, int64_t t, int64_t e) {
  return ((b * c.H_q + hq) * c.Nq + (t - c.q_t0)) * c.d + e;
}
int64_t kv_index(const Cfg& c, int64_t b, int64_t h, int64_t j, int64_t e) {
  return ((b * c.H_kv + h) * c.N + j) * c.d + e;
}

// Summary vector of block r at level l of head (b, h): level 0 is the raw
// key itself (k-bar^{(0)}_i = k_i, §Pyramid); higher levels read the fp64
// pyramid.
void summary(const Cfg& c, const void* k, const double* pyr, const std::vector<int64_t>& off,
             int64_t R, int64_t b, int64_t h, int64_t l, int64_t r, std::vector<double>& out) {
  out.resize(c.d);
  if (l == 0) {
    for (int64_t e = 0; e < c.d; ++e) out[e] = elem(k, kv_index(c, b, h, r, e), c.dtype);
  } else {
    const double* row = pyr + ((b * c.H_kv + h) * R + off[l] + r) * c.d;
    for (int64_t e = 0; e < c.d; ++e) out[e] = row[e];
  }
}

double dot_q(const Cfg& c, const void* q, int64_t b, int64_t hq, int64_t t, const std::vector<double>& v) {
  double s = 0;
  for (int64_t e = 0; e < c.d; ++e) s += elem(q, q_index(c, b, hq, t, e), c.dtype) * v[e];
  return s;
}

// Score of candidate block i at level l for kv head h and query t (§TopK LSE
// block score, summed over the GQA group as in §Kernels):
//   u = sum_{h' in group(h)} log sum_{r in Ch_{l-1}(i), r usable} exp(q_{h',t} . kbar^{(l-1)}_r * scale)
// At l = 1 the children are raw keys, so this is the exact block LSE.
// GQA reading (not stated on the page): query head h' belongs to kv head
// floor(h' / G_Q).
double block_score(const Cfg& c, const void* q, const void* k, const double* pyr,
                   const std::vector<int64_t>& M, const std::vector<int64_t>& off, int64_t R,
                   int64_t b, int64_t h, int64_t t, int64_t l, int64_t i) {
  const int64_t G = c.H_q / c.H_kv;
  const double sc = cfg_scale(c);
  std::vector<int64_t> ch;
  for (int64_t r : children(c, M, l, i))
    if (valid_block(c, M, l - 1, r, t)) ch.push_back(r);
  std::vector<std::vector<double>> sums(ch.size());
  for (size_t n = 0; n < ch.size(); ++n) summary(c, k, pyr, off, R, b, h, l - 1, ch[n], sums[n]);
  double u = 0;
  for (int64_t g = 0; g < G; ++g) {
    int64_t hq = h * G + g;
    std::vector<double> logits;
    for (size_t n = 0; n < ch.size(); ++n) logits.push_back(sc * dot_q(c, q, b, hq, t, sums[n]));
    u += logsumexp(logits);
  }
  return u;
}

// Keep the K best of (score, index) pairs: higher score first, equal scores
// to the lower block index (the page does not say how ties break). Returns
// the kept indices and the gap between the K-th and (K+1)-th scores.
std::vector<int64_t> top_k(std::vector<std::pair<double, int64_t>> v, int64_t K, double* gap) {
  std::sort(v.begin(), v.end(), [](const auto& a, const auto& b) {
    if (a.first != b.first) return a.first > b.first;
    return a.second < b.second;
  });
  *gap = v[K - 1].first - v[K].first;
  std::vector<int64_t> kept;
  for (int64_t n = 0; n < K; ++n) kept.push_back(v[n].second);
  return kept;
}

// Coarse-to-fine selection for one (b, kv head h, query t), §TopK:
//   A^{(L)} = {root}; at level l keep the valid candidates; if at most K are
//   valid keep them all unscored, else keep the top K by block_score; expand
//   the kept blocks to their children to form A^{(l-1)}; T = I^{(1)}.
// Writes K leaf indices ascending, -1 padded (the page treats T as a set).
// min_gap: smallest K-th minus (K+1)-th score over the scored levels.
// Optional trace (per level l = 0..L, 2K slots): valid candidates, their
// scores (NaN when the level was kept unscored) and whether each was kept.
void select_row(const Cfg& c, const void* q, const void* k, const double* pyr, int64_t b, int64_t h,
                int64_t t, int32_t* sel, double* min_gap, int32_t* tr_n, int32_t* tr_cand,
                double* tr_score, uint8_t* tr_kept) {
  const std::vector<int64_t> M = level_sizes(c.N, c.C);
  const std::vector<int64_t> off = level_offsets(M);
  const int64_t L = static_cast<int64_t>(M.size()) - 1;
  const int64_t R = off[L + 1];
  const int64_t W = 2 * c.K;
  *min_gap = std::numeric_limits<double>::infinity();
  std::vector<int64_t> A = {0};
  std::vector<int64_t> kept;
  for (int64_t l = L; l >= 1; --l) {
    std::vector<int64_t> V;
    for (int64_t i : A)
      if (valid_block(c, M, l, i, t)) V.push_back(i);
    std::vector<double> score(V.size(), std::numeric_limits<double>::quiet_NaN());
    if (static_cast<int64_t>(V.size()) <= c.K) {
      kept = V;  // at most K valid candidates: all kept without scoring
    } else {
      std::vector<std::pair<double, int64_t>> su;
      for (size_t n = 0; n < V.size(); ++n) {
        score[n] = block_score(c, q, k, pyr, M, off, R, b, h, t, l, V[n]);
        su.emplace_back(score[n], V[n]);
      }
      double gap;
      kept = top_k(su, c.K, &gap);
      *min_gap = std::min(*min_gap, gap);
    }
    if (tr_n) {
      tr_n[l] = static_cast<int32_t>(V.size());
      for (size_t n = 0; n < V.size() && static_cast<int64_t>(n) < W; ++n) {
        tr_cand[l * W + n] = static_cast<int32_t>(V[n]);
        tr_score[l * W + n] = score[n];
        tr_kept[l * W + n] = std::find(kept.begin(), kept.end(), V[n]) != kept.end();
      }
    }
    if (l > 1) {
      A.clear();
      for (int64_t i : kept)
        for (int64_t r : children(c, M, l, i)) A.push_back(r);
    }
  }
  std::sort(kept.begin(), kept.end());
  for (int64_t n = 0; n < c.K; ++n) sel[n] = n < static_cast<int64_t>(kept.size()) ? static_cast<int32_t>(kept[n]) : -1;
}

}  // namespace

extern "C" {

typedef Cfg oracle_cfg;

// Number of levels L and the row offset of each level (off[0..L]: level l
// starts at off[l-1]; off[L] = R rows per head). Returns L.
int64_t oracle_geometry(int64_t N, int64_t C, int64_t* sizes /*[L+1] or null*/, int64_t* offsets /*[L+1] or null*/) {
  std::vector<int64_t> M = level_sizes(N, C);
  std::vector<int64_t> off = level_offsets(M);
  int64_t L = static_cast<int64_t>(M.size()) - 1;
  if (sizes)
    for (int64_t l = 0; l <= L; ++l) sizes[l] = M[l];
  if (offsets)
    for (int64_t l = 0; l <= L; ++l) offsets[l] = off[l + 1];
  return L;
}

// §Pyramid mean pooling: leaves are the mean of their (up to C) raw keys;
// each higher block is the unweighted mean of its existing children,
// kbar^{(l+1)}_i = (1/|Ch_l(i)|) sum_{r in Ch_l(i)} kbar^{(l)}_r. A ragged last
// block is averaged over the children it has (reading: |Ch| counts existing
// children, not nominal ones). k: [B, H, N, d]; pyr: [B, H, R, d] fp64.
void oracle_build_pyramid(const void* k, int64_t dtype, int64_t B, int64_t H, int64_t N, int64_t d,
                          int64_t C, double* pyr) {
  const std::vector<int64_t> M = level_sizes(N, C);
  const std::vector<int64_t> off = level_offsets(M);
  const int64_t L = static_cast<int64_t>(M.size()) - 1;
  const int64_t R = off[L + 1];
#pragma omp parallel for schedule(dynamic)
  for (int64_t bh = 0; bh < B * H; ++bh) {
    double* P = pyr + bh * R * d;
    for (int64_t i = 0; i < M[1]; ++i) {
      int64_t lo = i * C, hi = std::min(lo + C, N);
      for (int64_t e = 0; e < d; ++e) {
        double s = 0;
        for (int64_t j = lo; j < hi; ++j) s += elem(k, (bh * N + j) * d + e, dtype);
        P[(off[1] + i) * d + e] = s / static_cast<double>(hi - lo);
      }
    }
    for (int64_t l = 1; l < L; ++l) {
      for (int64_t i = 0; i < M[l + 1]; ++i) {
        int64_t lo = 2 * i, hi = std::min(2 * i + 2, M[l]);
        for (int64_t e = 0; e < d; ++e) {
          double s = 0;
          for (int64_t r = lo; r < hi; ++r) s += P[(off[l] + r) * d + e];
          P[(off[l + 1] + i) * d + e] = s / static_cast<double>(hi - lo);
        }
      }
    }
  }
}

// Coarse-to-fine selection (§TopK) for a list of rows, each row a
// (b, kv head, t) triple. sel: [n, K]; min_gap: [n]. Trace buffers may be
// null; otherwise tr_n: [n, L+1], tr_cand/tr_score/tr_kept: [n, L+1, 2K].
void oracle_select_rows(const oracle_cfg* c, const void* q, const void* k, const double* pyr, int64_t n,
                        const int64_t* rows, int32_t* sel, double* min_gap, int32_t* tr_n, int32_t* tr_cand,
                        double* tr_score, uint8_t* tr_kept) {
  const int64_t L = static_cast<int64_t>(level_sizes(c->N, c->C).size()) - 1;
  const int64_t W = 2 * c->K;
#pragma omp parallel for schedule(dynamic)
  for (int64_t r = 0; r < n; ++r) {
    select_row(*c, q, k, pyr, rows[3 * r], rows[3 * r + 1], rows[3 * r + 2], sel + r * c->K, min_gap + r,
               tr_n ? tr_n + r * (L + 1) : nullptr, tr_cand ? tr_cand + r * (L + 1) * W : nullptr,
               tr_score ? tr_score + r * (L + 1) * W : nullptr, tr_kept ? tr_kept + r * (L + 1) * W : nullptr);
  }
}

// Flat single-level selector (§BSA: a flat method scores all M = ceil(N/C)
// block summaries per query). Reading of the summary score: the dot product
// of each query head with the leaf mean summary, scaled and summed over the
// GQA group: u_i = sum_{h'} scale * q_{h',t} . kbar^{(1)}_i. Same validity,
// keep-all, tie and output rules as the pyramid selector.
void oracle_select_flat_rows(const oracle_cfg* c, const void* q, const double* pyr, int64_t n,
                             const int64_t* rows, int32_t* sel, double* min_gap) {
  const std::vector<int64_t> M = level_sizes(c->N, c->C);
  const std::vector<int64_t> off = level_offsets(M);
  const int64_t L = static_cast<int64_t>(M.size()) - 1;
  const int64_t R = off[L + 1];
  const int64_t G = c->H_q / c->H_kv;
  const double sc = cfg_scale(*c);
#pragma omp parallel for schedule(dynamic)
  for (int64_t r = 0; r < n; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
    min_gap[r] = std::numeric_limits<double>::infinity();
    std::vector<int64_t> V;
    for (int64_t i = 0; i < M[1]; ++i)
      if (valid_block(*c, M, 1, i, t)) V.push_back(i);
    std::vector<int64_t> kept;
    if (static_cast<int64_t>(V.size()) <= c->K) {
      kept = V;
    } else {
      std::vector<std::pair<double, int64_t>> su;
      std::vector<double> s;
      for (int64_t i : V) {
        summary(*c, nullptr, pyr, off, R, b, h, 1, i, s);
        double u = 0;
        for (int64_t g = 0; g < G; ++g) u += sc * dot_q(*c, q, b, h * G + g, t, s);
        su.emplace_back(u, i);
      }
      kept = top_k(su, c->K, &min_gap[r]);
    }
    std::sort(kept.begin(), kept.end());
    for (int64_t m = 0; m < c->K; ++m)
      sel[r * c->K + m] = m < static_cast<int64_t>(kept.size()) ? static_cast<int32_t>(kept[m]) : -1;
  }
}

// Exact-score flat selector: the single-level block selection that the page
// contrasts PISA with (§BSA: a flat method scores every block of the sequence;
// §TopK: a block's score is the LSE of its raw keys). Every usable leaf gets
// the pyramid selector's own leaf-level score,
//   u_i = sum_{h' in group(h)} log sum_{j in leaf i, j usable} exp(scale q_{h',t} . k_j),
// with the same validity, keep-all, tie and output rules. This is what the
// coarse-to-fine search approximates: when the search scores every usable leaf
// (M_1 <= 2K) the two coincide.
void oracle_select_exact_rows(const oracle_cfg* c, const void* q, const void* k, int64_t n, const int64_t* rows,
                              int32_t* sel, double* min_gap) {
  const std::vector<int64_t> M = level_sizes(c->N, c->C);
  const std::vector<int64_t> off = level_offsets(M);
  const int64_t L = static_cast<int64_t>(M.size()) - 1;
  const int64_t R = off[L + 1];
#pragma omp parallel for schedule(dynamic)
  for (int64_t r = 0; r < n; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
    min_gap[r] = std::numeric_limits<double>::infinity();
    std::vector<int64_t> V;
    for (int64_t i = 0; i < M[1]; ++i)
      if (valid_block(*c, M, 1, i, t)) V.push_back(i);
    std::vector<int64_t> kept;
    if (static_cast<int64_t>(V.size()) <= c->K) {
      kept = V;
    } else {
      std::vector<std::pair<double, int64_t>> su;
      for (int64_t i : V) su.emplace_back(block_score(*c, q, k, nullptr, M, off, R, b, h, t, 1, i), i);
      kept = top_k(su, c->K, &min_gap[r]);
    }
    std::sort(kept.begin(), kept.end());
    for (int64_t m = 0; m < c->K; ++m)
      sel[r * c->K + m] = m < static_cast<int64_t>(kept.size()) ? static_cast<int32_t>(kept[m]) : -1;
  }
}

// Block-sparse attention (§BSA):
//   o_t = sum_{j in T_t} exp(q_t . k_j * scale) v_j / sum_{j in T_t} exp(q_t . k_j * scale)
// over the raw keys and values of the selected leaf blocks, for every query
// head of the kv head's group. T_t is the union of the selected blocks (sel
// entries < 0 are padding); under the causal reading only keys j <= t count.
// out: [n, G, d]; lse: [n, G] = log of the softmax denominator.
void oracle_attn_rows(const oracle_cfg* c, const void* q, const void* k, const void* v, int64_t n,
                      const int64_t* rows, const int32_t* sel, double* out, double* lse) {
  const int64_t G = c->H_q / c->H_kv;
  const double sc = cfg_scale(*c);
#pragma omp parallel for schedule(dynamic)
  for (int64_t r = 0; r < n; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
    std::vector<int64_t> keys;
    std::vector<int64_t> blocks;
    for (int64_t m = 0; m < c->K; ++m)
      if (sel[r * c->K + m] >= 0) blocks.push_back(sel[r * c->K + m]);
    std::sort(blocks.begin(), blocks.end());
    blocks.erase(std::unique(blocks.begin(), blocks.end()), blocks.end());
    for (int64_t i : blocks)
      for (int64_t j = i * c->C; j < std::min((i + 1) * c->C, c->N); ++j)
        if (!c->causal || j <= t) keys.push_back(j);
    for (int64_t g = 0; g < G; ++g) {
      const int64_t hq = h * G + g;
      std::vector<double> logit(keys.size());
      for (size_t n2 = 0; n2 < keys.size(); ++n2) {
        double s = 0;
        for (int64_t e = 0; e < c->d; ++e)
          s += elem(q, q_index(*c, b, hq, t, e), c->dtype) * elem(k, kv_index(*c, b, h, keys[n2], e), c->dtype);
        logit[n2] = sc * s;
      }
      const double z = logsumexp(logit);
      lse[r * G + g] = z;
      for (int64_t e = 0; e < c->d; ++e) {
        double acc = 0;
        for (size_t n2 = 0; n2 < keys.size(); ++n2)
          acc += std::exp(logit[n2] - z) * elem(v, kv_index(*c, b, h, keys[n2], e), c->dtype);
        out[(r * G + g) * c->d + e] = keys.empty() ? 0.0 : acc;
      }
    }
  }
}

// Gradient of the block-sparse attention (§BSA) with the selection held
// fixed: the selection is a discrete choice, so only the attention over the
// selected keys is differentiated. For every row (b, kv head h, t) and query
// head h' of the group, over the row's usable keys j (the union of its
// selected blocks; causal: j <= t), with dout the gradient of o:
//   s_j = scale q.k_j,  P_j = exp(s_j) / sum_i exp(s_i),  o = sum_j P_j v_j,
//   dP_j = dout . v_j,  D = dout . o,  dS_j = P_j (dP_j - D),
//   dq += scale sum_j dS_j k_j,  dk_j += scale dS_j q,  dv_j += P_j dout.
// Every row of the problem is processed (the key gradients sum over rows).
// q, dout: [B, H_q, N, d]; k, v: [B, H_kv, N, d]; sel: [B, H_kv, N, K].
// dq: [B, H_q, N, d]; dk, dv: [B, H_kv, N, d]; fp64, overwritten.
void oracle_attn_bwd(const oracle_cfg* c, const void* q, const void* k, const void* v, const int32_t* sel,
                     const void* dout, double* dq, double* dk, double* dv) {
  const int64_t G = c->H_q / c->H_kv;
  const double sc = cfg_scale(*c);
  const int64_t d = c->d;
  std::fill(dq, dq + c->B * c->H_q * c->N * d, 0.0);
  std::fill(dk, dk + c->B * c->H_kv * c->N * d, 0.0);
  std::fill(dv, dv + c->B * c->H_kv * c->N * d, 0.0);
#pragma omp parallel for schedule(dynamic)
  for (int64_t bh = 0; bh < c->B * c->H_kv; ++bh) {  // one kv head owns its dk, dv
    const int64_t b = bh / c->H_kv, h = bh % c->H_kv;
    for (int64_t t = 0; t < c->N; ++t) {
      const int32_t* srow = sel + (bh * c->N + t) * c->K;
      std::vector<int64_t> blocks;
      for (int64_t m = 0; m < c->K; ++m)
        if (srow[m] >= 0) blocks.push_back(srow[m]);
      std::sort(blocks.begin(), blocks.end());
      blocks.erase(std::unique(blocks.begin(), blocks.end()), blocks.end());
      std::vector<int64_t> keys;
      for (int64_t i : blocks)
        for (int64_t j = i * c->C; j < std::min((i + 1) * c->C, c->N); ++j)
          if (!c->causal || j <= t) keys.push_back(j);
      if (keys.empty()) continue;
      for (int64_t g = 0; g < G; ++g) {
        const int64_t hq = h * G + g;
        std::vector<double> qv(d), go(d), o(d, 0.0);
        for (int64_t e = 0; e < d; ++e) {
          qv[e] = elem(q, q_index(*c, b, hq, t, e), c->dtype);
          go[e] = elem(dout, q_index(*c, b, hq, t, e), c->dtype);
        }
        std::vector<double> logit(keys.size());
        for (size_t n2 = 0; n2 < keys.size(); ++n2) {
          double s = 0;
          for (int64_t e = 0; e < d; ++e) s += qv[e] * elem(k, kv_index(*c, b, h, keys[n2], e), c->dtype);
          logit[n2] = sc * s;
        }
        const double z = logsumexp(logit);
        std::vector<double> P(keys.size()), dP(keys.size());
        for (size_t n2 = 0; n2 < keys.size(); ++n2) {
          P[n2] = std::exp(logit[n2] - z);
          double dp = 0;
          for (int64_t e = 0; e < d; ++e) {
            const double ve = elem(v, kv_index(*c, b, h, keys[n2], e), c->dtype);
            o[e] += P[n2] * ve;
            dp += go[e] * ve;
          }
          dP[n2] = dp;
        }
        double D = 0;
        for (int64_t e = 0; e < d; ++e) D += go[e] * o[e];
        double* dqr = dq + ((b * c->H_q + hq) * c->N + t) * d;
        for (size_t n2 = 0; n2 < keys.size(); ++n2) {
          const double dS = P[n2] * (dP[n2] - D);
          double* dkr = dk + (bh * c->N + keys[n2]) * d;
          double* dvr = dv + (bh * c->N + keys[n2]) * d;
          for (int64_t e = 0; e < d; ++e) {
            dqr[e] += sc * dS * elem(k, kv_index(*c, b, h, keys[n2], e), c->dtype);
            dkr[e] += sc * dS * qv[e];
            dvr[e] += P[n2] * go[e];
          }
        }
      }
    }
  }
}

// dq of the attention backward for a list of rows only (a row's dq depends on
// that row alone): the same formulas as oracle_attn_bwd, restricted to the
// given (b, kv head, t) rows. sel: [n, K] the rows' selections; dout as q.
// dq: [n, G, d].
void oracle_attn_bwd_dq_rows(const oracle_cfg* c, const void* q, const void* k, const void* v, int64_t n,
                             const int64_t* rows, const int32_t* sel, const void* dout, double* dq) {
  const int64_t G = c->H_q / c->H_kv;
  const double sc = cfg_scale(*c);
  const int64_t d = c->d;
#pragma omp parallel for schedule(dynamic)
  for (int64_t r = 0; r < n; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
    std::vector<int64_t> blocks;
    for (int64_t m = 0; m < c->K; ++m)
      if (sel[r * c->K + m] >= 0) blocks.push_back(sel[r * c->K + m]);
    std::sort(blocks.begin(), blocks.end());
    blocks.erase(std::unique(blocks.begin(), blocks.end()), blocks.end());
    std::vector<int64_t> keys;
    for (int64_t i : blocks)
      for (int64_t j = i * c->C; j < std::min((i + 1) * c->C, c->N); ++j)
        if (!c->causal || j <= t) keys.push_back(j);
    for (int64_t g = 0; g < G; ++g) {
      double* out = dq + (r * G + g) * d;
      std::fill(out, out + d, 0.0);
      if (keys.empty()) continue;
      const int64_t hq = h * G + g;
      std::vector<double> qv(d), go(d), o(d, 0.0);
      for (int64_t e = 0; e < d; ++e) {
        qv[e] = elem(q, q_index(*c, b, hq, t, e), c->dtype);
        go[e] = elem(dout, q_index(*c, b, hq, t, e), c->dtype);
      }
      std::vector<double> logit(keys.size()), P(keys.size()), dP(keys.size());
      for (size_t n2 = 0; n2 < keys.size(); ++n2) {
        double s = 0;
        for (int64_t e = 0; e < d; ++e) s += qv[e] * elem(k, kv_index(*c, b, h, keys[n2], e), c->dtype);
        logit[n2] = sc * s;
      }
      const double z = logsumexp(logit);
      for (size_t n2 = 0; n2 < keys.size(); ++n2) {
        P[n2] = std::exp(logit[n2] - z);
        double dp = 0;
        for (int64_t e = 0; e < d; ++e) {
          const double ve = elem(v, kv_index(*c, b, h, keys[n2], e), c->dtype);
          o[e] += P[n2] * ve;
          dp += go[e] * ve;
        }
        dP[n2] = dp;
      }
      double D = 0;
      for (int64_t e = 0; e < d; ++e) D += go[e] * o[e];
      for (size_t n2 = 0; n2 < keys.size(); ++n2) {
        const double dS = P[n2] * (dP[n2] - D);
        for (int64_t e = 0; e < d; ++e) out[e] += sc * dS * elem(k, kv_index(*c, b, h, keys[n2], e), c->dtype);
      }
    }
  }
}

// Decode cache update (§Kernels, decoding paragraph: cache the mean pyramid
// and, per new token, update only the current leaf mean and its ancestor
// path). seq_keys: [n + 1, d] keys of one sequence and head, the new key last
// (position n). pyr: this sequence's pyramid for capacity `cap` tokens, laid
// out like oracle_build_pyramid for N = cap (level l at the offset it has for
// cap tokens); rows outside the first M_l(n + 1) of a level are not read.
void oracle_decode_append(const void* seq_keys, int64_t dtype, int64_t n, int64_t d, int64_t C, int64_t cap,
                          double* pyr) {
  const std::vector<int64_t> Mc = level_sizes(cap, C);
  const std::vector<int64_t> off = level_offsets(Mc);
  const std::vector<int64_t> M = level_sizes(n + 1, C);  // sizes after the append
  const int64_t L = static_cast<int64_t>(M.size()) - 1;
  // The leaf that holds key n: mean over the keys it holds now.
  int64_t leaf = n / C;
  for (int64_t e = 0; e < d; ++e) {
    double s = 0;
    for (int64_t j = leaf * C; j <= n; ++j) s += elem(seq_keys, j * d + e, dtype);
    pyr[(off[1] + leaf) * d + e] = s / static_cast<double>(n - leaf * C + 1);
  }
  // Its ancestors, one per level up to the (possibly new) root: the mean of
  // the children that exist after the append.
  int64_t node = leaf;
  for (int64_t l = 2; l <= L; ++l) {
    node /= 2;
    int64_t lo = 2 * node, hi = std::min(2 * node + 2, M[l - 1]);
    for (int64_t e = 0; e < d; ++e) {
      double s = 0;
      for (int64_t r = lo; r < hi; ++r) s += pyr[(off[l - 1] + r) * d + e];
      pyr[(off[l] + node) * d + e] = s / static_cast<double>(hi - lo);
    }
  }
}

}  // extern "C"
