#include "select2.cuh"

namespace pisa {

size_t select2_workspace_bytes(const PrefillArgs& a) { return 16; }

cudaError_t launch_select2(const PrefillArgs& a, const void* q, const void* k, const float* pyr, const Layout& lay,
                           int32_t* sel, float* sel_score, void* ws, cudaStream_t st) {
  return launch_select_rows(a, q, k, pyr, lay, sel, sel_score, st);
}

}  // namespace pisa
