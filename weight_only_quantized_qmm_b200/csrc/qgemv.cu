// Entry of the decode GEMV / MoE kernel family: picks the instantiation
// (bits, group size, dtype, token tiles, fused gate+up).  qgemv_b{2,3,4,6,8}.cu
// instantiate the kernels per bit width and try, in order: the streaming kernel
// (qgemv_stream.cuh: 2/4/8-bit whole-word lanes, rows of whole 128-byte slices,
// K / gs a multiple of 8), the per-warp TMA kernel (qgemv_tma.cuh: 2/4/8-bit
// whole-word shares, 16-byte rows), and the cp.async kernel (qgemv_impl.cuh:
// every other shape, including 3- and 6-bit codes).
#include <algorithm>

#include <cuda.h>

#include "qgemv.cuh"

namespace qmm {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link-time dependency on libcuda).
EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

cudaError_t launch_qgemv_b2(const QgemvParams&, int, int, int, bool, cudaStream_t);
cudaError_t launch_qgemv_b3(const QgemvParams&, int, int, int, bool, cudaStream_t);
cudaError_t launch_qgemv_b4(const QgemvParams&, int, int, int, bool, cudaStream_t);
cudaError_t launch_qgemv_b6(const QgemvParams&, int, int, int, bool, cudaStream_t);
cudaError_t launch_qgemv_b8(const QgemvParams&, int, int, int, bool, cudaStream_t);

constexpr int kMaxTokDispatch = 16;

cudaError_t launch_qgemv(QgemvParams prm, int bits, int gs, int dtype, bool dual,
                         cudaStream_t st) {
  const int tok_cap = prm.ids ? std::min(prm.n_pairs, kMaxTokDispatch) : prm.n_pairs;
  if (tok_cap <= 0) return cudaSuccess;
  if (tok_cap > kMaxTokDispatch) return cudaErrorInvalidValue;
  const int mt = tok_cap > 8 ? 2 : 1;
  switch (bits) {
    case 2: return launch_qgemv_b2(prm, gs, dtype, mt, dual, st);
    case 3: return launch_qgemv_b3(prm, gs, dtype, mt, dual, st);
    case 4: return launch_qgemv_b4(prm, gs, dtype, mt, dual, st);
    case 6: return launch_qgemv_b6(prm, gs, dtype, mt, dual, st);
    default: return launch_qgemv_b8(prm, gs, dtype, mt, dual, st);
  }
}

}  // namespace qmm
