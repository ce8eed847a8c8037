// Instantiations of the decode GEMV / MoE kernel family for 8-bit codes.
#include "qgemv_stream.cuh"

namespace qmm {

template <int GS, typename T>
static cudaError_t launch_tma_mt(const QgemvParams& prm, int64_t rows_total, int mt, bool dual,
                                 cudaStream_t st) {
  if (dual) {
    if (mt == 1) return launch_tma_one<8, GS, T, 1, true>(prm, rows_total, st);
    return launch_tma_one<8, GS, T, 2, true>(prm, rows_total, st);
  }
  if (mt == 1) return launch_tma_one<8, GS, T, 1, false>(prm, rows_total, st);
  return launch_tma_one<8, GS, T, 2, false>(prm, rows_total, st);
}

// TMA path when rows of packed words start on 16-byte boundaries and hold at
// least one 32-word box row; falls back to the cp.async path otherwise (or
// when the tensor map cannot be encoded).
static cudaError_t try_tma(const QgemvParams& prm, int gs, int dtype, int mt, bool dual,
                           cudaStream_t st) {
  const int64_t rows_total = prm.n_rows * prm.num_experts;
  if (prm.wpr % 4 != 0 || prm.wpr < 32 || rows_total < 16) return cudaErrorNotSupported;
  if (dtype == QMM_BF16) {
    if (gs == 32) return launch_tma_mt<32, __nv_bfloat16>(prm, rows_total, mt, dual, st);
    if (gs == 64) return launch_tma_mt<64, __nv_bfloat16>(prm, rows_total, mt, dual, st);
    return launch_tma_mt<128, __nv_bfloat16>(prm, rows_total, mt, dual, st);
  }
  if (gs == 32) return launch_tma_mt<32, __half>(prm, rows_total, mt, dual, st);
  if (gs == 64) return launch_tma_mt<64, __half>(prm, rows_total, mt, dual, st);
  return launch_tma_mt<128, __half>(prm, rows_total, mt, dual, st);
}

// per-tensor int8: 8-bit lanes (u = q + 128) in 64-code groups of 32-group
// units, one scale and bias for the tensor
template <typename T>
static cudaError_t launch_pt_t(const QgemvParams& prm, cudaStream_t st) {
  if (prm.n_pairs == 1) return stream::launch_stream<8, 64, T, 0, 32, 1, false, false, true>(prm, st);
  if (prm.n_pairs <= 8) return stream::launch_stream<8, 64, T, 1, 32, 1, false, false, true>(prm, st);
  if (prm.n_pairs <= 16) return stream::launch_stream<8, 64, T, 2, 32, 1, false, false, true>(prm, st);
  return cudaErrorNotSupported;
}

cudaError_t launch_qgemv_pt(const QgemvParams& prm, int dtype, cudaStream_t st) {
  if (dtype == QMM_BF16) return launch_pt_t<__nv_bfloat16>(prm, st);
  if (dtype == QMM_F16) return launch_pt_t<__half>(prm, st);
  return cudaErrorNotSupported;
}

cudaError_t launch_qgemv_b8(const QgemvParams& prm, int gs, int dtype, int mt, bool dual,
                            cudaStream_t st) {
  if (prm.use_tma) {
    const cudaError_t es = stream::try_stream<8>(prm, gs, dtype, mt, dual, st);
    if (es != cudaErrorNotSupported) return es;
    const cudaError_t e = try_tma(prm, gs, dtype, mt, dual, st);
    if (e != cudaErrorNotSupported) return e;
  }
  if (dtype == QMM_BF16) {
    if (gs == 32) return launch_mt<8, 32, __nv_bfloat16>(prm, mt, dual, st);
    if (gs == 64) return launch_mt<8, 64, __nv_bfloat16>(prm, mt, dual, st);
    return launch_mt<8, 128, __nv_bfloat16>(prm, mt, dual, st);
  }
  if (gs == 32) return launch_mt<8, 32, __half>(prm, mt, dual, st);
  if (gs == 64) return launch_mt<8, 64, __half>(prm, mt, dual, st);
  return launch_mt<8, 128, __half>(prm, mt, dual, st);
}

}  // namespace qmm
