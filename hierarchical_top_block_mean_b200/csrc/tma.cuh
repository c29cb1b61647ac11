// Tensor-memory-access (TMA) helpers: host-side tensor-map encoding and the
// device-side bulk tensor copy into shared memory with mbarrier completion.
//
// Every wait on an mbarrier is bounded in time (kWaitNs). A wait that runs
// out increments the device fault counter that pisa_device_faults reports,
// and the kernel carries on with whatever the buffer holds, so a lost copy
// shows up as a counted fault and wrong numbers, never as a hung GPU.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace pisa {

// ------------------------------------------------------------------ host
// Encodes a 2-D bf16 tensor map over a row-major [rows][cols] array with a
// box of box_rows x 64 columns (128 bytes, 128-byte swizzle). Out-of-range
// rows read as zero.
cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows);

// 3-D bf16 tensor map over [d2][d1][d0] (d0 innermost) with a box of
// 64 x box1 x box2 elements and 128-byte swizzle.
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                              uint32_t box1, uint32_t box2);
// 3-D bf16 map with explicit byte strides of dimensions 1 and 2 (any order of
// magnitude, e.g. a head dimension outside a token dimension), a box of
// 64 x box1 x box2 elements and 128-byte swizzle.
cudaError_t make_tmap_bf16_3d_strided(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                                      uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box1, uint32_t box2);

// Device address of the fault counter (bounded waits that ran out) on the
// current device; kernels that wait take it as an argument.
unsigned long long* wait_fault_counter();

// ------------------------------------------------------------------ device
__device__ inline uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ inline void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }

// Arrives once and adds `bytes` to the transaction count the phase waits for.
__device__ inline void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Tests the phase; while it is incomplete the thread may be suspended in
// hardware for a system-dependent time, so pollers do not steal issue slots.
__device__ inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity.
__device__ inline bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ inline uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s

// Waits for the phase with the given parity to complete; bounded in time.
__device__ inline bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long* faults) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitNs) {
      if ((threadIdx.x & 31) == 0 && faults) atomicAdd(faults, 1ull);
      return false;
    }
  }
  return true;
}

__device__ inline void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ inline void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ inline void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

// Orders this thread's earlier generic-proxy accesses to shared memory
// before later async-proxy (TMA) writes to it.
__device__ inline void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// Bulk tensor copy of one box at (x = column, y = row) into shared memory;
// completion is signalled on bar as transaction bytes. x * 2 bytes is a
// multiple of 16 at every call site (x is 0 or 64).
__device__ inline void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Byte offset of element (row, col) in a stack of 128-byte-swizzled boxes of
// box_rows rows x 64 bf16 columns (box b holds columns 64 b .. 64 b + 63).
template <int kBoxRows>
__device__ inline uint32_t swz128(int row, int col) {
  const int box = col >> 6, c16 = (col & 63) >> 3;
  return static_cast<uint32_t>(box * kBoxRows * 128 + row * 128 + ((c16 ^ (row & 7)) << 4) + ((col & 7) << 1));
}

}  // namespace pisa
