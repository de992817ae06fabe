// Device-side helpers shared by the libvq kernels: shared-memory addresses,
// mbarriers with bounded waits, 1-D bulk async copies (TMA engine, no tensor
// map, never multicast) and 128-bit shared-memory loads.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace vq {

// Device error word codes (bit flags, OR-ed by any CTA that hits one).
enum : uint32_t {
  kDevErrWaitTimeout = 1u,   // an mbarrier wait hit its iteration limit
  kDevErrBadShape = 2u,      // a kernel saw parameters its launcher should have rejected
};

// Error word every kernel may OR a flag into; read and cleared by
// vq_poll_device_error on the host. The library is one translation unit
// (vq_api.cu includes every kernel), so this definition exists once.
__device__ uint32_t g_device_error = 0;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make the initialised barrier visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for phase `parity` of `bar` with an iteration limit (each try_wait
// already suspends for a hardware-chosen time). Returns false on timeout after
// recording kDevErrWaitTimeout; the caller must then skip its dependent work
// but still take every barrier its CTA or cluster expects.
// The limit (2^25 polls, with a short sleep after the first 64) is seconds
// long: far beyond any legitimate wait inside one kernel, short enough to end a
// kernel whose producer never arrives.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t max_iters = (1u << 25)) {
  for (uint32_t it = 0; it < max_iters; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (it > 64) __nanosleep(100);
  }
  atomicOr(&g_device_error, kDevErrWaitTimeout);
  return false;
}

// The same wait by a whole warp, with one result for every lane.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity));
}

// 1-D bulk copy global -> this CTA's shared memory; completion is counted in
// bytes on `bar`. Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_addr(p)));
  return v;
}

}  // namespace vq
