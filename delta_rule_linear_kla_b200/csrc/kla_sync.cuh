// Bounded waits for the tensor-core kernels: every mbarrier wait gives up
// after about two seconds of %globaltimer instead of hanging the GPU.
#pragma once

#include <stdint.h>

#include "ptx_sm100.cuh"

namespace kla {

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Returns false if the phase with `parity` did not complete within
// `limit_ns` nanoseconds of %globaltimer.
__device__ __forceinline__ bool wait_bounded_ns(uint64_t* bar, uint32_t parity,
                                                uint64_t limit_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity) {
  return wait_bounded_ns(bar, parity, kWaitLimitNs);
}

}  // namespace kla
