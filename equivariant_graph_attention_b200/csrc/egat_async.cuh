// Asynchronous-copy building blocks of the egat kernels: mbarriers, 1-D bulk
// copies (cp.async.bulk: the TMA engine's untiled form, from this GPU's
// global memory into the CTA's own shared memory; never multicast), and
// bounded waits.
//
// Every wait on an mbarrier goes through bounded_wait: it gives up after a
// bounded number of polls, counts the give-up in this compilation unit's
// g_wait_timeouts (read and cleared through egat_take_device_status) and sets
// the CTA's abort flag, so that no launch can hang on a copy that never lands.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace egat {
namespace {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// mbarrier and bulk-copy (TMA engine, no multicast) helpers
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Waits of this compilation unit that gave up since the last
// egat_take_device_status (all launches on this device).
__device__ unsigned int g_wait_timeouts;
// Polls before a wait gives up.  try_wait suspends the thread for at most a
// hardware-defined interval per poll, so this bounds a wait to about a
// second; a stage's copies normally land within microseconds.
constexpr int kWaitPolls = 1 << 20;
constexpr int kDrainPolls = 1 << 14;

// Wait until the phase of parity `parity` of the mbarrier at `bar` has
// completed, polling at most `polls` times.  On giving up: count it, set the
// CTA's abort flag and return false; once the flag is set, a wait whose
// phase is not complete at the first poll returns at once, so a CTA whose
// copies never land finishes its loop (with meaningless results, reported by
// egat_take_device_status) instead of hanging.
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, int polls,
                                             volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;   // common case: no flag read
  if (*abort_flag) return false;
  for (int i = 1; i < polls; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  atomicAdd(&g_wait_timeouts, 1u);
  *abort_flag = 1;
  return false;
}
// Read and clear this compilation unit's give-up count (synchronises st).
inline int take_unit_wait_timeouts(cudaStream_t st, unsigned int* count) {
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_wait_timeouts) != cudaSuccess) return -3;   // EGAT_ERR_CUDA
  unsigned int h = 0;
  if (cudaMemcpyAsync(&h, addr, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(addr, 0, sizeof(h), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return -3;
  *count = h;
  return 0;
}

}  // namespace
}  // namespace egat
