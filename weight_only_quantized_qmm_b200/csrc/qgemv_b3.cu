// Instantiations of the decode GEMV / MoE kernel family for 3-bit codes.
#include "qgemv_stream.cuh"

namespace qmm {

cudaError_t launch_qgemv_b3(const QgemvParams& prm, int gs, int dtype, int mt, bool dual,
                            cudaStream_t st) {
  // the streaming kernel, else (shapes it does not take) the cp.async kernel
  if (prm.use_tma) {
    const cudaError_t es = stream::try_stream<3>(prm, gs, dtype, mt, dual, st);
    if (es != cudaErrorNotSupported) return es;
  }
  if (dtype == QMM_BF16) {
    if (gs == 32) return launch_mt<3, 32, __nv_bfloat16>(prm, mt, dual, st);
    if (gs == 64) return launch_mt<3, 64, __nv_bfloat16>(prm, mt, dual, st);
    return launch_mt<3, 128, __nv_bfloat16>(prm, mt, dual, st);
  }
  if (gs == 32) return launch_mt<3, 32, __half>(prm, mt, dual, st);
  if (gs == 64) return launch_mt<3, 64, __half>(prm, mt, dual, st);
  return launch_mt<3, 128, __half>(prm, mt, dual, st);
}

}  // namespace qmm
