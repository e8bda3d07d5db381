// A hint that pulls a byte range of global memory into L2 with the TMA
// engine (cp.async.bulk.prefetch.L2): no registers held and no completion to
// wait for, so a kernel can start its next tile's DRAM reads while it still
// works on the current one.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace ft {

// Ranges that are not 16-byte aligned are skipped (their loads then go to
// DRAM as they would without the hint); long ranges go out in 64 KB pieces.
__device__ __forceinline__ void l2_prefetch(const uint8_t* p, size_t bytes) {
  if ((reinterpret_cast<uintptr_t>(p) & 15) || (bytes & 15)) return;
  while (bytes > 0) {
    const uint32_t n = bytes > 65536 ? 65536u : (uint32_t)bytes;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(n) : "memory");
    p += n;
    bytes -= n;
  }
}

}  // namespace ft
