/*
 * pisa.h — C ABI of the B200 (sm_100a) PISA hot path: mean-pooled key
 * pyramid, coarse-to-fine top-K block selection, flat and exact-score
 * single-level block selection, block-sparse attention forward and backward,
 * query shards for sequence-parallel prefill, and the decode step over dense
 * or paged KV caches.
 *
 * The method is "Block Sparse Attention with Log-Linear Complexity"
 * (Tang, Qin, Pan, Li, Liu). Citations below name sections of its hyper.ai
 * page (the translated paper body): §BSA "Block-sparse attention",
 * §Pyramid "Pyramid key-block hierarchy", §TopK "Coarse-to-fine Top-K
 * selection", §Kernels "Kernel implementation", §Complexity.
 *
 * Conventions shared by every entry point
 *   - Pointers named q, k, v, pyr, sel, out, lse, ws, k_cache, v_cache, len,
 *     status are DEVICE pointers to memory the caller owns. The library never
 *     allocates, never synchronises the device and keeps no state between
 *     calls (except the launch counter of pisa_launch_count, the records of
 *     pisa_timing_start/stop and the scratch of pisa_select_noalloc).
 *   - Tensors are dense and row-major: q [B, H_q, N, d]; k, v [B, H_kv, N, d];
 *     query head h' belongs to kv head h' / G_Q with G_Q = H_q / H_kv.
 *   - dtype selects the storage of q, k, v and out: PISA_DTYPE_BF16 or
 *     PISA_DTYPE_F32. Pyramids are always fp32; lse is always fp32.
 *   - Blocks, levels and indices are 0-based (the paper's root block "1" is
 *     block 0 here). Level 1 holds the leaf blocks of C keys; level l >= 2
 *     merges pairs (g = 2) of level l-1.
 *   - Causal reading (the paper does not state one): a block is usable by
 *     the query at position t iff its first key is <= t; leaf scores and
 *     attention use only keys <= t.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All work is enqueued on it; results are ready when the stream is.
 *   - Arguments are validated on the host before anything is enqueued. A
 *     rejected call returns its error and enqueues nothing. A launch failure
 *     returns PISA_ERR_CUDA. Nothing in the library traps or waits without a
 *     bound.
 *   - Supported shapes: g = 2; C in {32, 64}; d in {64, 128}; 1 <= K <= 16;
 *     q_tile = 4; G_Q in {1, 2, 4, 8}; for the prefill calls also
 *     B * H_q * N < 2^31 and N < 2^27. Other values return
 *     PISA_ERR_UNSUPPORTED.
 */
#ifndef PISA_H_
#define PISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PISA_OK = 0,
  PISA_ERR_INVALID_ARGUMENT = 1, /* null pointer, non-positive size, H_q % H_kv != 0, ... */
  PISA_ERR_UNSUPPORTED = 2,      /* valid but outside the supported shapes listed above   */
  PISA_ERR_WORKSPACE = 3,        /* ws is null or smaller than pisa_select_workspace_bytes */
  PISA_ERR_CAPACITY = 4,         /* decode: a sequence is full (written to the status word) */
  PISA_ERR_CUDA = 5,             /* a CUDA launch or runtime call failed                   */
  PISA_ERR_DEVICE = 6            /* a device-side check failed (written to a status word)  */
} pisa_status;

typedef enum { PISA_DTYPE_F32 = 0, PISA_DTYPE_BF16 = 1 } pisa_dtype;

/* Prefill problem. scale <= 0 selects 1/sqrt(d) (§BSA). causal is 0 or 1. */
typedef struct {
  int32_t B, N, H_q, H_kv, d, C, g, K, q_tile, causal;
  int32_t dtype; /* pisa_dtype */
  float scale;
} pisa_config;

/* Decode problem: S independent sequences, each with room for cap tokens. */
typedef struct {
  int32_t S, cap, H_q, H_kv, d, C, g, K;
  int32_t dtype; /* pisa_dtype */
  float scale;
} pisa_decode_config;

/* Human-readable name of a status code (static storage). */
const char* pisa_status_string(int32_t status);

/* Library version as major * 10000 + minor * 100 + patch. */
int32_t pisa_version(void);

/* Number of kernels this library has launched in this process (all devices,
 * all entry points). Host-side counter; for accounting and tests. */
uint64_t pisa_launch_count(void);

/* Number of bounded device-side waits (on shared-memory copy barriers) that
 * ran out of time on the current device since the library was loaded. Each
 * such wait is abandoned after 2 s instead of hanging, so a non-zero count
 * means some outputs are wrong. Diagnostic only: this call synchronises the
 * device (it copies the counter to the host). Returns UINT64_MAX on error. */
uint64_t pisa_device_faults(void);

/*
 * Per-kernel timing for profiling. Not part of the method; a measurement aid.
 * After pisa_timing_start(), every kernel this library launches (on any
 * stream, from any entry point) is bracketed by two CUDA events recorded on
 * its launching stream, until pisa_timing_stop(). Each bracketed launch
 * creates two events, so keep timing windows short and off the hot path of
 * production runs; outside a window the cost is one atomic load per launch.
 *   pisa_timing_start: clears earlier records and turns timing on.
 *   pisa_timing_stop: turns timing off, waits for the recorded events (this
 *     synchronises with every stream that was timed), and writes up to
 *     max_kernels entries, one per kernel name in first-launch order:
 *     names[i] (a static string owned by the library), total_ms[i] (sum of
 *     event durations) and launches[i]. Any array may be NULL. Returns the
 *     number of distinct kernel names (which may exceed max_kernels), or -1
 *     if an event failed (the records are dropped either way).
 * Kernels overlapping on several streams are each timed from their own
 * stream's events, so their durations include any time shared with others.
 */
pisa_status pisa_timing_start(void);
int pisa_timing_stop(int max_kernels, const char** names, double* total_ms, int* launches);

/*
 * Pyramid geometry (host only, pure integer arithmetic) — §Pyramid level
 * sizes: M_0 = N, M_1 = ceil(N / C), M_{l+1} = ceil(M_l / g) until M_L = 1.
 * Writes L to *num_levels. If level_offsets is not NULL it receives L + 1
 * entries: level l (1..L) occupies rows [level_offsets[l-1], level_offsets[l])
 * of a head's pyramid, finest level first, and level_offsets[L] is the row
 * count R. Returns PISA_ERR_INVALID_ARGUMENT for N < 1, C < 1 or g != 2.
 */
pisa_status pisa_pyramid_geometry(int64_t N, int32_t C, int32_t g, int32_t* num_levels, int64_t* level_offsets);

/* Rows R of one head's pyramid for N tokens (0 on invalid input). */
int64_t pisa_pyramid_rows(int64_t N, int32_t C);

/*
 * Mean-pooled key pyramid — §Pyramid summary recursion: a leaf summary is the
 * mean of its (up to C) raw keys, every higher summary the unweighted mean of
 * the children the block has.
 *   k   : [B, H_kv, N, d] in cfg->dtype.
 *   pyr : [B, H_kv, R, d] fp32, R = pisa_pyramid_rows(N, C), laid out as in
 *         pisa_pyramid_geometry. Fully overwritten.
 */
pisa_status pisa_build_pyramid(const pisa_config* cfg, const void* k, float* pyr, void* stream);

/* Bytes of scratch workspace pisa_select needs for cfg (0 on invalid cfg). */
size_t pisa_select_workspace_bytes(const pisa_config* cfg);

/*
 * Coarse-to-fine top-K leaf-block selection — §TopK (candidate sets, keep-all
 * rule, LSE block score) with the GQA score sum and the two-stage split of
 * §Kernels: stage 1 routes levels L..2, stage 2 groups queries by candidate
 * leaf into tiles of q_tile queries, scores leaves by their exact raw-key LSE
 * and keeps the final top K. Ties go to the lower block index.
 *   q        : [B, H_q, N, d];  k : [B, H_kv, N, d];  pyr : from pisa_build_pyramid.
 *   sel      : [B, H_kv, N, K] int32 — selected leaf blocks per (kv head, query),
 *              ascending, padded with -1 when fewer than K blocks are valid.
 *   sel_score: NULL, or [B, H_kv, N, K] fp32 — the leaf-level score of each
 *              selected block (NaN when the leaf level was kept unscored, or
 *              for padding).
 *   ws       : device scratch of at least pisa_select_workspace_bytes(cfg)
 *              bytes, caller-owned, contents on entry ignored.
 */
pisa_status pisa_select(const pisa_config* cfg, const void* q, const void* k, const float* pyr, int32_t* sel,
                        float* sel_score, void* ws, size_t ws_bytes, void* stream);

/*
 * Flat single-level selection — §BSA: a flat method scores all M = ceil(N/C)
 * leaf summaries per query. Score reading: u_i = sum over the group of
 * scale * q_{h',t} . kbar^{(1)}_i; top K with the same validity, tie, order
 * and padding rules as pisa_select.
 *   q : [B, H_q, N, d];  pyr : [B, H_kv, R, d] (only level 1 is read);
 *   sel : [B, H_kv, N, K] int32.
 *   ws : device scratch of at least pisa_select_flat_workspace_bytes(cfg)
 *        bytes, 256-byte aligned, caller-owned, contents on entry ignored
 *        (bf16 with d = 128 needs it: the group-summed queries and the leaf
 *        summaries, each split into bf16 hi and lo planes; otherwise the size
 *        is 0 and ws may be NULL). Too small a ws returns PISA_ERR_WORKSPACE
 *        before anything is enqueued.
 */
size_t pisa_select_flat_workspace_bytes(const pisa_config* cfg);
pisa_status pisa_select_flat(const pisa_config* cfg, const void* q, const float* pyr, int32_t* sel, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * Exact-score flat selection — the single-level block selection that the
 * pyramid search approximates (§BSA: a flat method scores every block; §TopK:
 * a block's score is the LSE of its raw keys). Every usable leaf is scored by
 *   u_i = sum over the group of log sum_{j in leaf i, j usable} exp(scale q_{h',t} . k_j)
 * (the pyramid search's leaf-level score) and the top K are kept with the same
 * validity, keep-all, tie, order and padding rules as pisa_select. Work is
 * O(N^2 d) per kv head; needs no pyramid and no workspace.
 *   q : [B, H_q, N, d];  k : [B, H_kv, N, d];  sel : [B, H_kv, N, K] int32.
 * bf16 with d = 128 and C = 64 runs on tcgen05 tensor cores; other
 * configurations on a warp-per-row kernel.
 */
pisa_status pisa_select_exact(const pisa_config* cfg, const void* q, const void* k, int32_t* sel, void* stream);

/*
 * Block-sparse attention forward — §BSA:
 *   o_t = sum_{j in T_t} exp(scale q_t.k_j) v_j / sum_{j in T_t} exp(scale q_t.k_j)
 * over the raw keys of the selected leaf blocks T_t (shared by the query heads
 * of a GQA group; keys > t excluded when causal). Negative sel entries are
 * padding; the blocks of a row must be distinct, and every row must select at
 * least one usable block.
 *   sel : [B, H_kv, N, K] int32;  out : [B, H_q, N, d] in cfg->dtype;
 *   lse : NULL or [B, H_q, N] fp32, natural-log softmax denominator.
 *   ws  : NULL, or device scratch of at least pisa_attn_fwd_workspace_bytes(cfg)
 *         bytes, 256-byte aligned, caller-owned, contents on entry ignored.
 * With a workspace, bf16 problems with d = 128, C = 64 and G_Q in {4, 8} run
 * by leaf bucket: the selection is inverted per (kv head, query window, leaf),
 * each selected block's K and V are loaded once per tile of the queries that
 * chose it, each (query, block) pair leaves a partial softmax state
 * (max, sum, normalised output; about G_Q * 264 bytes) in the workspace, and
 * a merge pass combines every row's K partials in slot order. The workspace
 * is large (K partials per query row: about 18 GB at N = 262144, H_kv = 2,
 * G_Q = 8, K = 16). With ws = NULL (or for other shapes) every row streams
 * its own blocks, using no scratch. A non-NULL ws smaller than the size
 * returns PISA_ERR_WORKSPACE before anything is enqueued. Both routes give
 * the same results within the attention tolerance; each is deterministic.
 */
size_t pisa_attn_fwd_workspace_bytes(const pisa_config* cfg);
pisa_status pisa_sparse_attn_fwd(const pisa_config* cfg, const void* q, const void* k, const void* v,
                                 const int32_t* sel, void* out, float* lse, void* ws, size_t ws_bytes,
                                 void* stream);

/*
 * Size of the device array pisa_select_noalloc uses as its scratch: 64 MiB,
 * reserved on every GPU that loads this library until the process exits.
 */
#define PISA_SELECT_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * pisa_select without a caller workspace. The paper has no counterpart: this
 * is an interface for callers that cannot allocate device memory when they
 * select, such as a plugin that its host framework hands only input and
 * output buffers (no workspace hook), or a service whose memory pool owns the
 * whole GPU. The selection (and every argument except the workspace) is that
 * of pisa_select for bf16 inputs; the scratch lives in a library-owned device
 * array of PISA_SELECT_NOALLOC_SCRATCH_BYTES.
 *   - Returns PISA_ERR_WORKSPACE, enqueuing nothing, when the problem needs
 *     more scratch than that (pisa_select_workspace_bytes(cfg) tells how much);
 *     PISA_ERR_UNSUPPORTED for fp32 inputs, whose selection needs no scratch
 *     (call pisa_select with ws = NULL).
 *   - Calls no cudaMalloc or cudaFree and allocates nothing.
 *   - The first call on each device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     A call in a new context on that device (after cudaDeviceReset) looks it
 *     up again, so it too should come before any capture.
 *   - All calls in the process share the one array per device: calls whose
 *     execution overlaps on the GPU (different streams, or different host
 *     threads without ordering) race on it and give wrong selections. Order
 *     them on one stream. Each call clears what it needs zeroed itself.
 */
pisa_status pisa_select_noalloc(const pisa_config* cfg, const void* q, const void* k, const float* pyr, int32_t* sel,
                                float* sel_score, void* stream);

/*
 * Backward of the block-sparse attention over a fixed selection — the
 * gradient of pisa_sparse_attn_fwd with sel held constant (the selection is a
 * discrete choice; only the attention over the selected blocks' keys is
 * differentiated, §BSA). For a row (kv head, t) and a query head of the group,
 * over the usable keys j of the selected blocks (causal: j <= t):
 *   P_j = exp(scale q.k_j - lse), dP_j = dout.v_j, D = dout.out,
 *   dS_j = P_j (dP_j - D); dq = scale sum_j dS_j k_j,
 *   dk_j += scale dS_j q, dv_j += P_j dout (summed over rows and heads).
 *   q, out, dout : [B, H_q, N, d] bf16 (out and lse as the forward wrote them);
 *   k, v : [B, H_kv, N, d] bf16;  sel : [B, H_kv, N, K];  lse : [B, H_q, N];
 *   dq : [B, H_q, N, d] fp32;  dk, dv : [B, H_kv, N, d] fp32 (overwritten).
 * bf16 only (PISA_ERR_UNSUPPORTED otherwise). ws: at least
 * pisa_attn_bwd_workspace_bytes(cfg) bytes, 16-byte aligned, else
 * PISA_ERR_WORKSPACE. dk and dv are accumulated with atomics, so they are
 * reproducible only up to fp32 rounding order.
 */
size_t pisa_attn_bwd_workspace_bytes(const pisa_config* cfg);
pisa_status pisa_sparse_attn_bwd(const pisa_config* cfg, const void* q, const void* k, const void* v,
                                 const int32_t* sel, const void* out, const float* lse, const void* dout, float* dq,
                                 float* dk, float* dv, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------ query shards
 * Sequence-parallel prefill. Split one sequence's queries by position over
 * several GPUs, so that each GPU computes only its own rows' selection and
 * attention. Each query row's selection and attention depend only on that
 * row and on the keys (§TopK, §BSA), so a shard gives bit-for-bit the rows
 * that the whole-sequence call gives. The keys, the values and the pyramid
 * are the whole sequence's; every GPU holds a full copy of them, and the
 * caller gathers them, for instance with an NCCL all-gather of the
 * per-GPU key and value slices.
 *
 * A shard covers query positions [q0, q0 + n_q) of the N-token sequence that
 * cfg describes (0 <= q0, 1 <= n_q, q0 + n_q <= N; else
 * PISA_ERR_INVALID_ARGUMENT). These arrays hold the shard's rows only:
 *   q         : [B, H_q, n_q, d];  out : [B, H_q, n_q, d];  lse : [B, H_q, n_q]
 *   sel       : [B, H_kv, n_q, K];  sel_score : [B, H_kv, n_q, K]
 * These arrays hold all N positions, as in the whole-sequence calls:
 *   k, v : [B, H_kv, N, d];  pyr : from pisa_build_pyramid over all N keys.
 * Row j of a shard is the query at position q0 + j. It sees keys <= q0 + j
 * when causal, and all N keys otherwise. Other arguments, error codes and
 * ownership are those of pisa_select and pisa_sparse_attn_fwd;
 * {q0 = 0, n_q = N} is exactly those calls.
 */
typedef struct {
  int32_t q0, n_q;
} pisa_query_span;

/* Scratch bytes pisa_select_span needs: it scales with n_q, not N. Returns
 * 0 for an invalid cfg or span, and for fp32, which needs none. */
size_t pisa_select_span_workspace_bytes(const pisa_config* cfg, const pisa_query_span* span);
pisa_status pisa_select_span(const pisa_config* cfg, const pisa_query_span* span, const void* q, const void* k,
                             const float* pyr, int32_t* sel, float* sel_score, void* ws, size_t ws_bytes,
                             void* stream);
/* Scratch bytes of the bucketed attention for a shard (0 when that route
 * does not apply to cfg, or for an invalid span). */
size_t pisa_attn_fwd_span_workspace_bytes(const pisa_config* cfg, const pisa_query_span* span);
pisa_status pisa_sparse_attn_fwd_span(const pisa_config* cfg, const pisa_query_span* span, const void* q,
                                      const void* k, const void* v, const int32_t* sel, void* out, float* lse,
                                      void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- decode
 * §Kernels, decoding: the mean pyramid is cached; per new token only the
 * current leaf mean and its ancestor path are updated, and one fused kernel
 * selects from the coarsest level down to the leaves, scoring raw key blocks
 * directly.
 *   k_cache, v_cache : [S, H_kv, cap, d] in dtype.
 *   pyr              : [S, H_kv, R_cap, d] fp32, R_cap = pisa_decode_pyramid_rows;
 *                      level l of every sequence sits at the offset it has for
 *                      cap tokens (pisa_pyramid_geometry(cap, ...)).
 *   len              : [S] int32 device, tokens held per sequence.
 *   status           : one int32 device word; kernels store PISA_ERR_CAPACITY
 *                      there when a sequence is full (that sequence is skipped)
 *                      and never clear it.
 */
int64_t pisa_decode_pyramid_rows(const pisa_decode_config* cfg);

/* Bytes of device workspace that pisa_decode_attn and pisa_decode_step need
 * (0 when the configuration needs none; 0 also for an invalid cfg). The
 * fused kernel keeps there, per (sequence, kv head), the scaled logits
 * scale q.k of the keys of up to 2K leaf blocks (fp32, [2K][C][G_Q]), so the
 * attention reuses the leaf scorer's products instead of reading K again.
 * Owned by the caller; contents need no initialisation and are scratch. */
int64_t pisa_decode_workspace_bytes(const pisa_decode_config* cfg);

/* Builds every sequence's pyramid over its first len[s] cached keys. */
pisa_status pisa_decode_init(const pisa_decode_config* cfg, const void* k_cache, float* pyr, const int32_t* len,
                             void* stream);

/* Appends k_new/v_new [S, H_kv, d] at position len[s], updates that leaf
 * mean and its ancestors, then increments len[s]. */
pisa_status pisa_decode_append(const pisa_decode_config* cfg, const void* k_new, const void* v_new, void* k_cache,
                               void* v_cache, float* pyr, int32_t* len, int32_t* status, void* stream);

/* Selects K leaf blocks for q_new [S, H_q, d], the query at position
 * len[s] - 1 (every block of the sequence is valid). sel: [S, H_kv, K]. */
pisa_status pisa_decode_select(const pisa_decode_config* cfg, const void* q_new, const void* k_cache,
                               const float* pyr, const int32_t* len, int32_t* sel, void* stream);

/* Attention of q_new over the selected blocks of each sequence's first
 * len[s] tokens. out: [S, H_q, d] in dtype; lse: NULL or [S, H_q] fp32.
 * workspace: pisa_decode_workspace_bytes(cfg) bytes of device memory,
 * 16-byte aligned (PISA_ERR_WORKSPACE when missing and needed). */
pisa_status pisa_decode_attn(const pisa_decode_config* cfg, const void* q_new, const void* k_cache,
                             const void* v_cache, const int32_t* len, const int32_t* sel, void* out, float* lse,
                             void* workspace, void* stream);

/* One decode step in one launch: append, select and attend for every
 * sequence. sel may be NULL (selection kept on chip); otherwise [S, H_kv, K].
 * workspace: as for pisa_decode_attn. */
pisa_status pisa_decode_step(const pisa_decode_config* cfg, const void* q_new, const void* k_new, const void* v_new,
                             void* k_cache, void* v_cache, float* pyr, int32_t* len, int32_t* sel, void* out,
                             float* lse, int32_t* status, void* workspace, void* stream);

/* ------------------------------------------------------ paged decode
 * The same decode path over KV caches held in fixed-size pages, as serving
 * systems keep them: one page holds one leaf block (C tokens) of one sequence
 * for every kv head.
 *   k_pages, v_pages : [num_pages, H_kv, C, d] in dtype (bf16 only);
 *   block_table      : [S, max_pages] int32 device; entry i is the page of
 *                      leaf i of the sequence, -1 where none is assigned.
 *                      Every other entry must be a page of the pool
 *                      (0 <= entry < num_pages): the library does not know
 *                      num_pages and cannot check it, so an entry out of range
 *                      makes the kernels read and write outside the pool;
 *   cfg->cap         : must equal max_pages * C.
 * Pages of the leaves a sequence already holds must be assigned. A step whose
 * new token falls in a leaf without a page stores PISA_ERR_CAPACITY in status
 * and skips that sequence, as a full dense cache does. Results are bit-for-bit
 * those of the dense calls on the same data. Other arguments as for
 * pisa_decode_init and pisa_decode_step; PISA_ERR_UNSUPPORTED when the
 * configuration has no fused kernel (see pisa_decode_step). */
pisa_status pisa_decode_init_paged(const pisa_decode_config* cfg, const void* k_pages, const int32_t* block_table,
                                   int max_pages, float* pyr, const int32_t* len, void* stream);
pisa_status pisa_decode_step_paged(const pisa_decode_config* cfg, const void* q_new, const void* k_new,
                                   const void* v_new, void* k_pages, void* v_pages, const int32_t* block_table,
                                   int max_pages, float* pyr, int32_t* len, int32_t* sel, void* out, float* lse,
                                   int32_t* status, void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PISA_H_ */
