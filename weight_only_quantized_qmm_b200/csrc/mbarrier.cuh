// Shared-memory mbarrier primitives of the CUDA path (sm_100a), used by the
// TMA-fed kernels for their pipelines.  Every wait is bounded: it polls a
// given number of times (each try_wait may suspend the thread for a while)
// and then reports failure instead of spinning on, so that a copy that never
// lands ends the kernel with a status rather than a hung GPU.
#pragma once

#include <stdint.h>

namespace qmm {

// Default poll limit of a pipeline wait (with the try_wait suspend hint this
// is far beyond any legitimate wait, and still ends in well under a second).
constexpr uint32_t kMbarSpins = 1u << 20;

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
// True once the phase with the given parity has completed.  A fresh barrier
// is in phase 0, so parity 1 (the phase "before" it) reads as completed.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
// Bounded wait: true when the phase completed within `spins` polls.
__device__ __forceinline__ bool mbar_wait_n(uint32_t bar, uint32_t parity, uint32_t spins) {
  for (uint32_t i = 0; i < spins; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
// Bounded wait that also gives up (false) as soon as another role of the CTA
// has raised *abort_flag (polled every 1024 tries).
__device__ __forceinline__ bool mbar_wait_abortable(uint32_t bar, uint32_t parity, uint32_t spins,
                                                    const int* abort_flag) {
  for (uint32_t i = 0; i < spins; ++i) {
    if ((i & 1023u) == 1023u && *reinterpret_cast<const volatile int*>(abort_flag)) return false;
    if (mbar_try_wait(bar, parity)) return true;
  }
  return false;
}

}  // namespace qmm
