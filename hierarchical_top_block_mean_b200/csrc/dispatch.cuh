// Compile-time dispatch over storage type, head dim and group size.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace pisa {

template <typename T>
struct TypeTag {
  using type = T;
};
template <int V>
using IntTag = std::integral_constant<int, V>;

// Calls f(TypeTag<T>{}, IntTag<D>{}) for the supported (dtype, d) pairs.
template <class F>
cudaError_t dispatch_td(int dtype, int d, F&& f) {
  if (dtype == PISA_DTYPE_BF16) {
    if (d == 128) return f(TypeTag<bf16>{}, IntTag<128>{});
    return f(TypeTag<bf16>{}, IntTag<64>{});
  }
  if (d == 128) return f(TypeTag<float>{}, IntTag<128>{});
  return f(TypeTag<float>{}, IntTag<64>{});
}

// Calls f(TypeTag<T>{}, IntTag<D>{}, IntTag<G>{}) for G in {1, 2, 4, 8}.
template <class F>
cudaError_t dispatch_tdg(int dtype, int d, int G, F&& f) {
  return dispatch_td(dtype, d, [&](auto tt, auto dd) -> cudaError_t {
    switch (G) {
      case 1: return f(tt, dd, IntTag<1>{});
      case 2: return f(tt, dd, IntTag<2>{});
      case 4: return f(tt, dd, IntTag<4>{});
      default: return f(tt, dd, IntTag<8>{});
    }
  });
}

// Copies the level offsets of a layout into shared memory (kernel params
// cannot be indexed dynamically without a local copy).
__device__ inline void load_offsets(const Layout& lay, int64_t* off) {
  for (int i = threadIdx.x; i < kMaxLevels + 2; i += blockDim.x) off[i] = lay.off[i];
  __syncthreads();
}

}  // namespace pisa
