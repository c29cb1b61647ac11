// pisa_select_noalloc: the bf16 two-stage selection of pisa_select, with its
// scratch taken from a fixed array that this library owns in device memory
// instead of from a caller workspace.
//
// Who needs it: callers that cannot call cudaMalloc (or hand out temporary
// device memory) when they select, e.g. a plugin whose host framework passes
// it only input and output buffers and offers no workspace hook, or a service
// whose memory pool owns the whole GPU and forbids allocations outside it.
//
// Cost: the array below is reserved on every GPU that loads this library and
// stays reserved until the process exits.
#include <mutex>

#include "select2.cuh"

namespace pisa {
pisa_status validate_prefill(const pisa_config* cfg);
}

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(PISA_SELECT_NOALLOC_SCRATCH_BYTES);
static_assert(kScratchBytes % 256 == 0, "scratch size keeps 256-byte sections aligned");

// The scratch itself. In host code this name is only a stand-in for the
// device symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_select_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_setup_mu;
void* g_scratch_dev[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};  // the context each cached address belongs to

// The current driver context (CUcontext) as an opaque handle, fetched through
// the runtime's driver entry point so that the library need not link libcuda.
void* current_context() {
  using Fn = int (*)(void**);
  static Fn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<Fn>(p);
  }();
  void* ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the scratch array on the current device. It is looked up
// with cudaGetSymbolAddress on the first call per device, with that device
// current, and cached. A new context on that device (after cudaDeviceReset
// the module is loaded again, possibly elsewhere) triggers a fresh lookup.
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_dev[dev] == nullptr || ctx == nullptr || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_dev[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" pisa_status pisa_select_noalloc(const pisa_config* cfg, const void* q, const void* k, const float* pyr,
                                           int32_t* sel, float* sel_score, void* stream) {
  using namespace pisa;
  const pisa_status s = validate_prefill(cfg);
  if (s != PISA_OK) return s;
  if (cfg->dtype != PISA_DTYPE_BF16) return PISA_ERR_UNSUPPORTED;  // fp32 selection uses no scratch
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!q || !k || !pyr || !sel || !al16(q) || !al16(k) || !al16(pyr) || !al16(sel))
    return PISA_ERR_INVALID_ARGUMENT;
  PrefillArgs a{cfg->B, cfg->N, cfg->H_q, cfg->H_kv, cfg->d, cfg->C, cfg->K, cfg->causal, cfg->dtype, cfg->scale,
                0, cfg->N};
  if (!(a.scale > 0.f)) a.scale = 1.0f / sqrtf(static_cast<float>(cfg->d));
  if (select2_workspace_bytes(a) > kScratchBytes) return PISA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return PISA_ERR_CUDA;
  const Layout lay = make_layout(cfg->N, cfg->C);
  const cudaError_t e =
      launch_select2(a, q, k, pyr, lay, sel, sel_score, scratch, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PISA_OK : PISA_ERR_CUDA;
}
