// Launchers behind the C ABI. Every launcher enqueues on `st`, counts its
// launches and returns the launch status; none synchronises or allocates.
#pragma once

#include "common.cuh"

namespace pisa {

// Prefill problem with the scale resolved (kernel parameter, passed by value).
struct PrefillArgs {
  int B, N, H_q, H_kv, d, C, K, causal, dtype;
  float scale;
  // Query rows of the q, sel, out and lse arrays: positions [q0, q0 + Nq)
  // of the N-key sequence (a whole sequence: q0 = 0, Nq = N). The
  // selection and forward attention kernels honour them; the flat, exact and
  // backward kernels take whole sequences only.
  int q0, Nq;
};

// Decode problem with the scale resolved.
struct DecodeArgs {
  int S, cap, H_q, H_kv, d, C, K, dtype;
  float scale;
};

// ---- warp-per-row kernels (fp32 path)
cudaError_t launch_select_rows(const PrefillArgs& a, const void* q, const void* k, const float* pyr,
                               const Layout& lay, int32_t* sel, float* sel_score, cudaStream_t st);
cudaError_t launch_attn_rows(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                             void* out, float* lse, cudaStream_t st);
cudaError_t launch_flat_rows(const PrefillArgs& a, const void* q, const float* pyr, int64_t R, int32_t* sel,
                             cudaStream_t st);

// ---- tensor-core attention (bf16)
cudaError_t launch_attn_mma(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                            void* out, float* lse, cudaStream_t st);
// Attention by leaf bucket (tcgen05; bf16, d = 128, C = 64, G_Q in {4, 8}):
// partial softmax states per (query, block) pair in ws, then a merge.
bool attn_bucket_supported(const PrefillArgs& a);
size_t attn_bucket_workspace_bytes(const PrefillArgs& a);
cudaError_t launch_attn_bucket(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                               void* out, float* lse, void* ws, cudaStream_t st);

cudaError_t launch_flat_mma(const PrefillArgs& a, const void* q, const float* pyr, int64_t R, int32_t* sel,
                            cudaStream_t st);
// tcgen05 flat selection (bf16, d = 128) with its hi/lo operand planes in ws.
bool flat_umma_supported(const PrefillArgs& a);
size_t flat_umma_workspace_bytes(const PrefillArgs& a);
cudaError_t launch_flat_umma(const PrefillArgs& a, const void* q, const float* pyr, int64_t R, int32_t* sel, void* ws,
                             cudaStream_t st);

// ---- decode
cudaError_t launch_decode_append(const DecodeArgs& a, const Layout& lay, const void* k_new, const void* v_new,
                                 void* k_cache, void* v_cache, float* pyr, int32_t* len, int32_t* status,
                                 cudaStream_t st);
// mode bit 1: select (writes sel if not null), bit 2: attend (reads sel from
// memory when bit 1 is clear).
cudaError_t launch_decode_rows(const DecodeArgs& a, const Layout& lay, int mode, const void* q_new,
                               const void* k_cache, const void* v_cache, const float* pyr, const int32_t* len,
                               int32_t* sel, void* out, float* lse, cudaStream_t st);

// ---- attention backward over a fixed selection (bf16 inputs, fp32 gradients)
size_t attn_bwd_workspace_bytes(const PrefillArgs& a);
cudaError_t launch_attn_bwd(const PrefillArgs& a, const void* q, const void* k, const void* v, const int32_t* sel,
                            const void* out, const float* lse, const void* dout, float* dq, float* dk, float* dv,
                            void* ws, cudaStream_t st);

// ---- exact-score flat selection (every usable leaf scored by its raw-key LSE)
cudaError_t launch_exact_rows(const PrefillArgs& a, const void* q, const void* k, int32_t* sel, cudaStream_t st);
bool exact_umma_supported(const PrefillArgs& a);
cudaError_t launch_exact_umma(const PrefillArgs& a, const void* q, const void* k, int32_t* sel, cudaStream_t st);

// Fused decode (bf16, H_kv <= 8, G_Q <= 8). mode bits: 1 append, 2 select, 4 attend.
// lgt_ws: decode_logit_floats(a) floats, required when attending. With a
// block table the caches are pages [num_pages][H_kv][C][d], page
// block_table[s * max_pages + i] holding leaf i of sequence s (cap = max_pages C).
bool decode_fused_supported(const DecodeArgs& a);
int64_t decode_logit_floats(const DecodeArgs& a);
cudaError_t launch_decode_fused(const DecodeArgs& a, const Layout& lay, int mode, const void* q_new,
                                const void* k_new, const void* v_new, void* k_cache, void* v_cache, float* pyr,
                                int32_t* len, int32_t* sel, void* out, float* lse, int32_t* status, float* lgt_ws,
                                cudaStream_t st, const int32_t* block_table = nullptr, int max_pages = 0);

}  // namespace pisa
