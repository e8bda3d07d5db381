// Shared-memory mbarriers and bulk asynchronous copies (the TMA engine) used
// by the producer/consumer pipelines of the expert kernels. Every wait is
// bounded: a wait that runs out raises the CTA's abort flag and latches
// DERR_TIMEOUT, so a kernel never spins forever.
#pragma once

#include "ft_internal.cuh"

namespace ft {
namespace mb {

constexpr long long WAIT_CYCLES = 4000000000ll;  // ~2 s at 2 GHz

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// Make barrier initialisation visible to the async proxy before first use.
__device__ __forceinline__ void fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `bar` with the given parity. Returns false
// (raising *abort and the device error) if it does not complete in time, or
// at once if the CTA already aborted.
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, volatile int* abort, uint32_t* err) {
  const long long t0 = clock64();
  for (uint32_t i = 0;; ++i) {
    if (try_wait(bar, parity)) return true;
    if ((i & 255) == 255) {
      if (*abort) return false;
      if (clock64() - t0 > WAIT_CYCLES) {
        *abort = 1;
        atomicExch(err, (uint32_t)DERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Wait without raising anything (used to drain in-flight copies on exit).
__device__ __forceinline__ void wait_quiet(uint32_t bar, uint32_t parity, long long cycles) {
  const long long t0 = clock64();
  while (!try_wait(bar, parity) && clock64() - t0 < cycles) {
  }
}

// Contiguous global -> shared copy by the TMA engine, completing `bytes` on
// `bar`. dst, src and bytes must be multiples of 16. No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

}  // namespace mb
}  // namespace ft
