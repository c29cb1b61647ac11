// C ABI entry points (include/pisa.h): host-side validation, layout
// arithmetic and dispatch to the kernels. Nothing here allocates device
// memory or synchronises; the only state is the launch counter.
#include <atomic>
#include <cmath>

#include "kernels.cuh"
#include "pyramid.cuh"
#include "select2.cuh"
#include "tma.cuh"

namespace pisa {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

namespace {

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline pisa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PISA_OK : PISA_ERR_CUDA; }

pisa_status check_shape(int H_q, int H_kv, int d, int C, int g, int K, int dtype) {
  if (H_q < 1 || H_kv < 1 || d < 1 || C < 1 || K < 1) return PISA_ERR_INVALID_ARGUMENT;
  if (H_q % H_kv != 0) return PISA_ERR_INVALID_ARGUMENT;
  if (dtype != PISA_DTYPE_F32 && dtype != PISA_DTYPE_BF16) return PISA_ERR_INVALID_ARGUMENT;
  const int G = H_q / H_kv;
  if (g != 2 || (C != 32 && C != 64) || (d != 64 && d != 128) || K > kMaxK) return PISA_ERR_UNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PISA_ERR_UNSUPPORTED;
  return PISA_OK;
}

pisa_status check_cfg(const pisa_config* c) {
  if (!c) return PISA_ERR_INVALID_ARGUMENT;
  if (c->B < 1 || c->N < 1 || (c->causal != 0 && c->causal != 1)) return PISA_ERR_INVALID_ARGUMENT;
  pisa_status s = check_shape(c->H_q, c->H_kv, c->d, c->C, c->g, c->K, c->dtype);
  if (s != PISA_OK) return s;
  if (c->q_tile != 4) return PISA_ERR_UNSUPPORTED;
  // Tensor-map row coordinates are 32-bit, and a stage-2 pair packs its query
  // position into 27 bits.
  if (static_cast<int64_t>(c->B) * c->H_q * c->N >= (int64_t{1} << 31) || c->N >= (1 << 27))
    return PISA_ERR_UNSUPPORTED;
  return PISA_OK;
}

pisa_status check_dcfg(const pisa_decode_config* c) {
  if (!c) return PISA_ERR_INVALID_ARGUMENT;
  if (c->S < 1 || c->cap < 1) return PISA_ERR_INVALID_ARGUMENT;
  return check_shape(c->H_q, c->H_kv, c->d, c->C, c->g, c->K, c->dtype);
}

PrefillArgs args_of(const pisa_config* c) {
  PrefillArgs a{c->B, c->N, c->H_q, c->H_kv, c->d, c->C, c->K, c->causal, c->dtype, c->scale, 0, c->N};
  if (!(a.scale > 0.f)) a.scale = 1.0f / std::sqrt(static_cast<float>(c->d));
  return a;
}

// Query span check; narrows a to the span's rows.
pisa_status apply_span(const pisa_query_span* sp, int N, PrefillArgs* a) {
  if (!sp || sp->q0 < 0 || sp->n_q < 1 || static_cast<int64_t>(sp->q0) + sp->n_q > N) return PISA_ERR_INVALID_ARGUMENT;
  a->q0 = sp->q0;
  a->Nq = sp->n_q;
  return PISA_OK;
}

DecodeArgs dargs_of(const pisa_decode_config* c) {
  DecodeArgs a{c->S, c->cap, c->H_q, c->H_kv, c->d, c->C, c->K, c->dtype, c->scale};
  if (!(a.scale > 0.f)) a.scale = 1.0f / std::sqrt(static_cast<float>(c->d));
  return a;
}

}  // namespace

// Argument check shared with entry points defined in other files.
pisa_status validate_prefill(const pisa_config* cfg) { return check_cfg(cfg); }

}  // namespace pisa

using namespace pisa;

extern "C" {

const char* pisa_status_string(int32_t status) {
  switch (status) {
    case PISA_OK: return "PISA_OK";
    case PISA_ERR_INVALID_ARGUMENT: return "PISA_ERR_INVALID_ARGUMENT";
    case PISA_ERR_UNSUPPORTED: return "PISA_ERR_UNSUPPORTED";
    case PISA_ERR_WORKSPACE: return "PISA_ERR_WORKSPACE";
    case PISA_ERR_CAPACITY: return "PISA_ERR_CAPACITY";
    case PISA_ERR_CUDA: return "PISA_ERR_CUDA";
    case PISA_ERR_DEVICE: return "PISA_ERR_DEVICE";
    default: return "PISA_ERR_UNKNOWN";
  }
}

int32_t pisa_version(void) { return 100; }

uint64_t pisa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

uint64_t pisa_device_faults(void) {
  unsigned long long* p = wait_fault_counter();
  unsigned long long v = 0;
  if (!p || cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return UINT64_MAX;
  return v;
}

pisa_status pisa_pyramid_geometry(int64_t N, int32_t C, int32_t g, int32_t* num_levels_out, int64_t* level_offsets) {
  if (N < 1 || C < 1 || g != 2 || !num_levels_out) return PISA_ERR_INVALID_ARGUMENT;
  const int L = num_levels(N, C);
  *num_levels_out = L;
  if (level_offsets) {
    int64_t acc = 0;
    for (int l = 1; l <= L; ++l) {
      level_offsets[l - 1] = acc;
      acc += level_size(N, C, l);
    }
    level_offsets[L] = acc;
  }
  return PISA_OK;
}

int64_t pisa_pyramid_rows(int64_t N, int32_t C) {
  if (N < 1 || C < 1) return 0;
  return make_layout(N, C).R;
}

pisa_status pisa_build_pyramid(const pisa_config* cfg, const void* k, float* pyr, void* stream) {
  pisa_status s = check_cfg(cfg);
  if (s != PISA_OK) return s;
  if (!k || !pyr || !aligned16(k) || !aligned16(pyr)) return PISA_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(cfg->N, cfg->C);
  return from_cuda(launch_build_pyramid(cfg->dtype, cfg->d, k, pyr, lay, cfg->N, cfg->N, nullptr,
                                        cfg->B * cfg->H_kv, cfg->H_kv, cfg->N, cfg->C, as_stream(stream)));
}

size_t pisa_select_span_workspace_bytes(const pisa_config* cfg, const pisa_query_span* span) {
  if (check_cfg(cfg) != PISA_OK) return 0;
  if (cfg->dtype != PISA_DTYPE_BF16) return 0;  // the fp32 path selects row by row without scratch
  PrefillArgs a = args_of(cfg);
  if (apply_span(span, cfg->N, &a) != PISA_OK) return 0;
  return select2_workspace_bytes(a);
}

size_t pisa_select_workspace_bytes(const pisa_config* cfg) {
  if (check_cfg(cfg) != PISA_OK) return 0;
  const pisa_query_span all{0, cfg->N};
  return pisa_select_span_workspace_bytes(cfg, &all);
}

pisa_status pisa_select_span(const pisa_config* cfg, const pisa_query_span* span, const void* q, const void* k,
                             const float* pyr, int32_t* sel, float* sel_score, void* ws, size_t ws_bytes,
                             void* stream) {
  pisa_status s = check_cfg(cfg);
  if (s != PISA_OK) return s;
  if (!q || !k || !pyr || !sel || !aligned16(q) || !aligned16(k) || !aligned16(pyr) || !aligned16(sel))
    return PISA_ERR_INVALID_ARGUMENT;
  PrefillArgs a = args_of(cfg);
  if ((s = apply_span(span, cfg->N, &a)) != PISA_OK) return s;
  const Layout lay = make_layout(cfg->N, cfg->C);
  if (cfg->dtype == PISA_DTYPE_BF16) {
    const size_t need = select2_workspace_bytes(a);
    if (!ws || ws_bytes < need || !aligned16(ws)) return PISA_ERR_WORKSPACE;
    return from_cuda(launch_select2(a, q, k, pyr, lay, sel, sel_score, ws, as_stream(stream)));
  }
  return from_cuda(launch_select_rows(a, q, k, pyr, lay, sel, sel_score, as_stream(stream)));
}

pisa_status pisa_select(const pisa_config* cfg, const void* q, const void* k, const float* pyr, int32_t* sel,
                        float* sel_score, void* ws, size_t ws_bytes, void* stream) {
  pisa_status s = check_cfg(cfg);
  if (s != PISA_OK) return s;
  const pisa_query_span all{0, cfg->N};
  return pisa_select_span(cfg, &all, q, k, pyr, sel, sel_score, ws, ws_bytes, stream);
}

size_t pisa_select_flat_workspace_bytes(const pisa_config* cfg) {
  if (check_cfg(cfg) != PISA_OK) return 0;
  return flat_umma_workspace_bytes(args_of(cfg));
}

pisa_status pisa_select_flat(const pisa_config* cfg, const void* q, const float* pyr, int32_t* sel, void* ws,
                             size_t ws_bytes, void* stream) {
  pisa_status s = check_cfg(cfg);
  if (s != PISA_OK) return s;
  if (!q || !pyr || !sel || !aligned16(q) || !aligned16(pyr) || !aligned16(sel)) return PISA_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(cfg->N, cfg->C);
  const PrefillArgs a = args_of(cfg);
  if (flat_umma_supported(a)) {
    const size_t need = flat_umma_workspace_bytes(a);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PISA_ERR_WORKSPACE;
    return from_cuda(launch_flat_umma(a, q, pyr, lay.R, sel, ws, as_stream(stream)));
  }
  if (cfg->dtype == PISA_DTYPE_BF16) return from_cuda(launch_flat_mma(a, q, pyr, lay.R, sel, as_stream(stream)));
  return from_cuda(launch_flat_rows(a, q, pyr, lay.R, sel, as_stream(stream)));
}

pisa_status pisa_select_exact(const pisa_config* cfg, const void* q, const void* k, int32_t* sel, void* stream) {
  pisa_status s = check_cfg(cfg);
  if (s != PISA_OK) return s;
  if (!q || !k || !sel || !aligned16(q) || !aligned16(k) || !aligned16(sel)) return PISA_ERR_INVALID_ARGUMENT;
  const PrefillArgs a = args_of(cfg);
  if (exact_umma_supported(a)) return from_cuda(launch_exact_umma(a, q, k, sel, as_stream(stream)));
  return from_cuda(launch_exact_rows(a, q, k, sel, as_stream(stream)));
}

size_t pisa_attn_fwd_span_workspace_bytes(const pisa_config* cfg, const pisa_query_span* span) {
  if (check_cfg(cfg) != PISA_OK) return 0;
  PrefillArgs a = args_of(cfg);
  if (apply_span(span, cfg->N, &a) != PISA_OK) return 0;
  return attn_bucket_workspace_bytes(a);
}

size_t pisa_attn_fwd_workspace_bytes(const pisa_config* cfg) {
  if (check_cfg(cfg) != PISA_OK) return 0;
  const pisa_query_span all{0, cfg->N};
  return pisa_attn_fwd_span_workspace_bytes(cfg, &all);
}

pisa_status pisa_sparse_attn_fwd_span(const pisa_config* cfg, const pisa_query_span* span, const void* q,
                                      const void* k, const void* v, const int32_t* sel, void* out, float* lse,
                                      void* ws, size_t ws_bytes, void* stream) {
  pisa_status s = check_cfg(cfg);
  if (s != PISA_OK) return s;
  if (!q || !k || !v || !sel || !out) return PISA_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return PISA_ERR_INVALID_ARGUMENT;
  PrefillArgs a = args_of(cfg);
  if ((s = apply_span(span, cfg->N, &a)) != PISA_OK) return s;
  if (ws && attn_bucket_supported(a)) {
    if (ws_bytes < attn_bucket_workspace_bytes(a) || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
      return PISA_ERR_WORKSPACE;
    return from_cuda(launch_attn_bucket(a, q, k, v, sel, out, lse, ws, as_stream(stream)));
  }
  if (cfg->dtype == PISA_DTYPE_BF16) return from_cuda(launch_attn_mma(a, q, k, v, sel, out, lse, as_stream(stream)));
  return from_cuda(launch_attn_rows(a, q, k, v, sel, out, lse, as_stream(stream)));
}

pisa_status pisa_sparse_attn_fwd(const pisa_config* cfg, const void* q, const void* k, const void* v,
                                 const int32_t* sel, void* out, float* lse, void* ws, size_t ws_bytes,
                                 void* stream) {
  pisa_status s = check_cfg(cfg);
  if (s != PISA_OK) return s;
  const pisa_query_span all{0, cfg->N};
  return pisa_sparse_attn_fwd_span(cfg, &all, q, k, v, sel, out, lse, ws, ws_bytes, stream);
}

size_t pisa_attn_bwd_workspace_bytes(const pisa_config* cfg) {
  if (check_cfg(cfg) != PISA_OK) return 0;
  return attn_bwd_workspace_bytes(args_of(cfg));
}

pisa_status pisa_sparse_attn_bwd(const pisa_config* cfg, const void* q, const void* k, const void* v,
                                 const int32_t* sel, const void* out, const float* lse, const void* dout, float* dq,
                                 float* dk, float* dv, void* ws, size_t ws_bytes, void* stream) {
  pisa_status s = check_cfg(cfg);
  if (s != PISA_OK) return s;
  if (cfg->dtype != PISA_DTYPE_BF16) return PISA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !sel || !out || !lse || !dout || !dq || !dk || !dv) return PISA_ERR_INVALID_ARGUMENT;
  for (const void* p : {q, k, v, out, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                        static_cast<const void*>(dv)})
    if (!aligned16(p)) return PISA_ERR_INVALID_ARGUMENT;
  const PrefillArgs a = args_of(cfg);
  if (!ws || !aligned16(ws) || ws_bytes < attn_bwd_workspace_bytes(a)) return PISA_ERR_WORKSPACE;
  return from_cuda(launch_attn_bwd(a, q, k, v, sel, out, lse, dout, dq, dk, dv, ws, as_stream(stream)));
}

int64_t pisa_decode_pyramid_rows(const pisa_decode_config* cfg) {
  if (check_dcfg(cfg) != PISA_OK) return 0;
  return make_layout(cfg->cap, cfg->C).R;
}

int64_t pisa_decode_workspace_bytes(const pisa_decode_config* cfg) {
  if (check_dcfg(cfg) != PISA_OK) return 0;
  const DecodeArgs a = dargs_of(cfg);
  return decode_fused_supported(a) ? decode_logit_floats(a) * 4 : 0;
}

pisa_status pisa_decode_init(const pisa_decode_config* cfg, const void* k_cache, float* pyr, const int32_t* len,
                             void* stream) {
  pisa_status s = check_dcfg(cfg);
  if (s != PISA_OK) return s;
  if (!k_cache || !pyr || !len || !aligned16(k_cache) || !aligned16(pyr)) return PISA_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(cfg->cap, cfg->C);
  return from_cuda(launch_build_pyramid(cfg->dtype, cfg->d, k_cache, pyr, lay, cfg->cap, 0, len,
                                        cfg->S * cfg->H_kv, cfg->H_kv, cfg->cap, cfg->C, as_stream(stream)));
}

namespace {
// Paged caches: fused path only, one leaf block per page, cap = max_pages * C.
pisa_status check_paged(const pisa_decode_config* cfg, const int32_t* block_table, int max_pages) {
  pisa_status s = check_dcfg(cfg);
  if (s != PISA_OK) return s;
  if (!block_table || max_pages < 1 || static_cast<int64_t>(max_pages) * cfg->C != cfg->cap)
    return PISA_ERR_INVALID_ARGUMENT;
  if (!decode_fused_supported(dargs_of(cfg))) return PISA_ERR_UNSUPPORTED;
  return PISA_OK;
}
}  // namespace

pisa_status pisa_decode_init_paged(const pisa_decode_config* cfg, const void* k_pages, const int32_t* block_table,
                                   int max_pages, float* pyr, const int32_t* len, void* stream) {
  pisa_status s = check_paged(cfg, block_table, max_pages);
  if (s != PISA_OK) return s;
  if (!k_pages || !pyr || !len || !aligned16(k_pages) || !aligned16(pyr)) return PISA_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(cfg->cap, cfg->C);
  return from_cuda(launch_build_pyramid(cfg->dtype, cfg->d, k_pages, pyr, lay, cfg->cap, 0, len,
                                        cfg->S * cfg->H_kv, cfg->H_kv, cfg->cap, cfg->C, as_stream(stream),
                                        PageMap{block_table, max_pages}));
}

pisa_status pisa_decode_step_paged(const pisa_decode_config* cfg, const void* q_new, const void* k_new,
                                   const void* v_new, void* k_pages, void* v_pages, const int32_t* block_table,
                                   int max_pages, float* pyr, int32_t* len, int32_t* sel, void* out, float* lse,
                                   int32_t* status, void* workspace, void* stream) {
  pisa_status s = check_paged(cfg, block_table, max_pages);
  if (s != PISA_OK) return s;
  if (!q_new || !k_new || !v_new || !k_pages || !v_pages || !pyr || !len || !out || !status)
    return PISA_ERR_INVALID_ARGUMENT;
  if (!aligned16(q_new) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(pyr))
    return PISA_ERR_INVALID_ARGUMENT;
  if (!workspace || !aligned16(workspace)) return PISA_ERR_WORKSPACE;
  const Layout lay = make_layout(cfg->cap, cfg->C);
  return from_cuda(launch_decode_fused(dargs_of(cfg), lay, 7, q_new, k_new, v_new, k_pages, v_pages, pyr, len, sel,
                                       out, lse, status, static_cast<float*>(workspace), as_stream(stream),
                                       block_table, max_pages));
}

pisa_status pisa_decode_append(const pisa_decode_config* cfg, const void* k_new, const void* v_new, void* k_cache,
                               void* v_cache, float* pyr, int32_t* len, int32_t* status, void* stream) {
  pisa_status s = check_dcfg(cfg);
  if (s != PISA_OK) return s;
  if (!k_new || !v_new || !k_cache || !v_cache || !pyr || !len || !status) return PISA_ERR_INVALID_ARGUMENT;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(pyr)) return PISA_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(cfg->cap, cfg->C);
  const DecodeArgs a = dargs_of(cfg);
  if (decode_fused_supported(a))
    return from_cuda(launch_decode_fused(a, lay, 1, nullptr, k_new, v_new, k_cache, v_cache, pyr, len, nullptr, nullptr,
                                         nullptr, status, nullptr, as_stream(stream)));
  return from_cuda(launch_decode_append(a, lay, k_new, v_new, k_cache, v_cache, pyr, len, status, as_stream(stream)));
}

pisa_status pisa_decode_select(const pisa_decode_config* cfg, const void* q_new, const void* k_cache,
                               const float* pyr, const int32_t* len, int32_t* sel, void* stream) {
  pisa_status s = check_dcfg(cfg);
  if (s != PISA_OK) return s;
  if (!q_new || !k_cache || !pyr || !len || !sel) return PISA_ERR_INVALID_ARGUMENT;
  if (!aligned16(q_new) || !aligned16(k_cache) || !aligned16(pyr)) return PISA_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(cfg->cap, cfg->C);
  const DecodeArgs a = dargs_of(cfg);
  if (decode_fused_supported(a))
    return from_cuda(launch_decode_fused(a, lay, 2, q_new, nullptr, nullptr, const_cast<void*>(k_cache),
                                         const_cast<void*>(k_cache), const_cast<float*>(pyr),
                                         const_cast<int32_t*>(len), sel, nullptr, nullptr, nullptr, nullptr,
                                         as_stream(stream)));
  return from_cuda(launch_decode_rows(a, lay, 1, q_new, k_cache, nullptr, pyr, len, sel, nullptr, nullptr,
                                      as_stream(stream)));
}

pisa_status pisa_decode_attn(const pisa_decode_config* cfg, const void* q_new, const void* k_cache,
                             const void* v_cache, const int32_t* len, const int32_t* sel, void* out, float* lse,
                             void* workspace, void* stream) {
  pisa_status s = check_dcfg(cfg);
  if (s != PISA_OK) return s;
  if (!q_new || !k_cache || !v_cache || !len || !sel || !out) return PISA_ERR_INVALID_ARGUMENT;
  if (!aligned16(q_new) || !aligned16(k_cache) || !aligned16(v_cache)) return PISA_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(cfg->cap, cfg->C);
  const DecodeArgs a = dargs_of(cfg);
  if (decode_fused_supported(a)) {
    if (!workspace || !aligned16(workspace)) return PISA_ERR_WORKSPACE;
    return from_cuda(launch_decode_fused(a, lay, 4, q_new, nullptr, nullptr, const_cast<void*>(k_cache),
                                         const_cast<void*>(v_cache), nullptr, const_cast<int32_t*>(len),
                                         const_cast<int32_t*>(sel), out, lse, nullptr,
                                         static_cast<float*>(workspace), as_stream(stream)));
  }
  return from_cuda(launch_decode_rows(a, lay, 2, q_new, k_cache, v_cache, nullptr, len, const_cast<int32_t*>(sel),
                                      out, lse, as_stream(stream)));
}

pisa_status pisa_decode_step(const pisa_decode_config* cfg, const void* q_new, const void* k_new, const void* v_new,
                             void* k_cache, void* v_cache, float* pyr, int32_t* len, int32_t* sel, void* out,
                             float* lse, int32_t* status, void* workspace, void* stream) {
  pisa_status s = check_dcfg(cfg);
  if (s != PISA_OK) return s;
  if (!q_new || !k_new || !v_new || !k_cache || !v_cache || !pyr || !len || !out || !status)
    return PISA_ERR_INVALID_ARGUMENT;
  if (!aligned16(q_new) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(pyr))
    return PISA_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(cfg->cap, cfg->C);
  const DecodeArgs a = dargs_of(cfg);
  if (decode_fused_supported(a)) {
    if (!workspace || !aligned16(workspace)) return PISA_ERR_WORKSPACE;
    return from_cuda(launch_decode_fused(a, lay, 7, q_new, k_new, v_new, k_cache, v_cache, pyr, len, sel, out, lse,
                                         status, static_cast<float*>(workspace), as_stream(stream)));
  }
  cudaError_t e = launch_decode_append(a, lay, k_new, v_new, k_cache, v_cache, pyr, len, status, as_stream(stream));
  if (e != cudaSuccess) return PISA_ERR_CUDA;
  return from_cuda(
      launch_decode_rows(a, lay, 3, q_new, k_cache, v_cache, pyr, len, sel, out, lse, as_stream(stream)));
}

}  // extern "C"
