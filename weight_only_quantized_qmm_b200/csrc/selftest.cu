// Diagnostic entry point: exercises the bounded mbarrier waits that every
// TMA-fed kernel of the library relies on, on a barrier that nothing ever
// arrives on, so that the give-up path (status QMM_ERR_TIMEOUT instead of a
// hung GPU) can be tested without breaking a real kernel.  No copy is in
// flight at any point: the kernel touches only its own shared memory.
#include "common.cuh"
#include "mbarrier.cuh"

namespace qmm {

__global__ void bounded_wait_selftest_kernel(uint32_t spins, int32_t* d_result, int32_t* d_status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 1;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the phase before the first one reads as completed: returns at once
    const bool before = mbar_wait_n(b, 1u, 1u);
    // phase 0 never completes (no arrival): the wait gives up after `spins` polls
    const bool pending = mbar_wait_n(b, 0u, spins);
    // with the abort flag raised, the abortable wait gives up within 1024 polls
    const bool aborted = mbar_wait_abortable(b, 0u, 0xFFFFFFFFu, &abort_flag);
    d_result[0] = before ? 1 : 0;
    d_result[1] = pending ? 1 : 0;
    d_result[2] = aborted ? 1 : 0;
    if (!pending) set_status(d_status, QMM_ERR_TIMEOUT);
  }
}

}  // namespace qmm

extern "C" qmm_status qmm_selftest_bounded_wait(uint32_t spins, int32_t* d_result, int32_t* d_status,
                                                void* stream) {
  if (spins == 0 || spins > (1u << 22)) return QMM_ERR_INVALID_ARG;
  const uintptr_t r = reinterpret_cast<uintptr_t>(d_result), s = reinterpret_cast<uintptr_t>(d_status);
  if (!d_result || (r & 3u) || !d_status || (s & 3u)) return QMM_ERR_ALIGNMENT;
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return QMM_ERR_CUDA;
  if (major != 10) return QMM_ERR_UNSUPPORTED;
  qmm::bounded_wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(spins, d_result, d_status);
  return cudaGetLastError() == cudaSuccess ? QMM_OK : QMM_ERR_CUDA;
}
