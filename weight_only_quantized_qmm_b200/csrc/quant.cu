// Affine quantize (dense -> packed codes, scales, biases) and standalone
// dequantize.
//
// Packing follows "emily 0.5.1 lib/emily/quantization.ex" (dequantize_defn/1:
// code i at stream bit i*bits, LSB-first, uint32 words, straddling for 3 and
// 6 bits).  The quantizer is the per-group min/max rule of
// "mlex 0.1.3 src/quant.rs" quantize_dynamic_int8 (EPSILON floor, round half
// away from zero) applied to each group of group_size columns.  Both kernels
// are bit-exact: the same fp32 operations in the same order as the
// definition (explicit _rn intrinsics so nothing is contracted).
#include <float.h>

#include "common.cuh"

namespace qmm {

// One thread per (row, group).  Untimed preparation step: the loads are
// strided across threads, but every 32-byte sector is reused from L1.
template <typename TW, typename TS, int B>
__global__ void __launch_bounds__(256)
quantize_kernel(const TW* __restrict__ w, int64_t rows, int64_t cols, int gs,
                uint32_t* __restrict__ packed, TS* __restrict__ scales, TS* __restrict__ biases) {
  const int64_t G = cols / gs;
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (idx >= rows * G) return;
  const int64_t r = idx / G, g = idx % G;
  const TW* src = w + r * cols + g * gs;
  const float qmax = (float)((1 << B) - 1);

  float mn = to_f32(src[0]), mx = mn;
  for (int i = 1; i < gs; ++i) {
    const float v = to_f32(src[i]);
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  float scale_f = __fdiv_rn(__fsub_rn(mx, mn), qmax);
  if (scale_f < FLT_EPSILON) scale_f = FLT_EPSILON;
  const TS s_st = from_f32<TS>(scale_f);
  const TS b_st = from_f32<TS>(__fadd_rn(mn, 0.0f));  // +0 turns -0 into +0
  scales[idx] = s_st;
  biases[idx] = b_st;
  const float s = to_f32(s_st), b = to_f32(b_st);

  // the group occupies exactly gs*B/32 whole words (gs*B is a multiple of 32)
  uint32_t words[32];
  const int nw = gs * B / 32;
#pragma unroll
  for (int i = 0; i < 32; ++i) words[i] = 0u;
  for (int i = 0; i < gs; ++i) {
    const float v = to_f32(src[i]);
    float q = roundf(__fdiv_rn(__fsub_rn(v, b), s));
    if (q < 0.0f) q = 0.0f;
    if (q > qmax) q = qmax;
    const uint32_t code = (uint32_t)q;
    const int p = i * B, wi = p >> 5, sh = p & 31;
    words[wi] |= code << sh;
    if (sh + B > 32) words[wi + 1] |= code >> (32 - sh);
  }
  uint32_t* dst = packed + r * (cols * B / 32) + g * nw;
  for (int i = 0; i < nw; ++i) dst[i] = words[i];
}

// One thread per 32 consecutive codes of a row (= B whole words, inside one
// group since group_size >= 32).  w_hat = fmaf(q, s, b), stored as TO.
template <int B, typename TS, typename TO>
__global__ void __launch_bounds__(256)
dequant_kernel(const uint32_t* __restrict__ packed, const TS* __restrict__ scales,
               const TS* __restrict__ biases, int64_t rows, int64_t cols, int gs,
               TO* __restrict__ out) {
  const int64_t chunks = cols / 32;
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (idx >= rows * chunks) return;
  const int64_t r = idx / chunks, c = idx % chunks;
  const int64_t G = cols / gs;
  const uint32_t* src = packed + r * (cols * B / 32) + c * B;
  uint32_t wr[B + 1];
#pragma unroll
  for (int i = 0; i < B; ++i) wr[i] = __ldg(src + i);
  wr[B] = 0u;
  const int64_t g = (c * 32) / gs;
  const float s = to_f32(scales[r * G + g]);
  const float b = to_f32(biases[r * G + g]);
  TO vals[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) vals[i] = from_f32<TO>(fmaf((float)stream_code<B>(wr, i), s, b));
  uint4* dst = reinterpret_cast<uint4*>(out + r * cols + c * 32);
  const uint4* v4 = reinterpret_cast<const uint4*>(vals);
#pragma unroll
  for (int i = 0; i < (int)(32 * sizeof(TO) / 16); ++i) dst[i] = v4[i];
}

// ------------------------------------------------------------------ launchers
template <typename TW, typename TS>
static cudaError_t launch_quant_b(int bits, const void* w, int64_t rows, int64_t cols, int gs,
                                  uint32_t* packed, void* scales, void* biases,
                                  cudaStream_t st) {
  const int64_t n = rows * (cols / gs);
  const int blocks = (int)((n + 255) / 256);
  auto W = reinterpret_cast<const TW*>(w);
  auto S = reinterpret_cast<TS*>(scales);
  auto Bi = reinterpret_cast<TS*>(biases);
  switch (bits) {
    case 2: quantize_kernel<TW, TS, 2><<<blocks, 256, 0, st>>>(W, rows, cols, gs, packed, S, Bi); break;
    case 3: quantize_kernel<TW, TS, 3><<<blocks, 256, 0, st>>>(W, rows, cols, gs, packed, S, Bi); break;
    case 4: quantize_kernel<TW, TS, 4><<<blocks, 256, 0, st>>>(W, rows, cols, gs, packed, S, Bi); break;
    case 6: quantize_kernel<TW, TS, 6><<<blocks, 256, 0, st>>>(W, rows, cols, gs, packed, S, Bi); break;
    default: quantize_kernel<TW, TS, 8><<<blocks, 256, 0, st>>>(W, rows, cols, gs, packed, S, Bi); break;
  }
  return cudaGetLastError();
}

template <typename TW>
static cudaError_t launch_quant_s(int s_dtype, int bits, const void* w, int64_t rows,
                                  int64_t cols, int gs, uint32_t* packed, void* scales,
                                  void* biases, cudaStream_t st) {
  if (s_dtype == QMM_F32)
    return launch_quant_b<TW, float>(bits, w, rows, cols, gs, packed, scales, biases, st);
  if (s_dtype == QMM_BF16)
    return launch_quant_b<TW, __nv_bfloat16>(bits, w, rows, cols, gs, packed, scales, biases, st);
  return launch_quant_b<TW, __half>(bits, w, rows, cols, gs, packed, scales, biases, st);
}

cudaError_t launch_quantize(int w_dtype, int s_dtype, int bits, const void* w, int64_t rows,
                            int64_t cols, int gs, uint32_t* packed, void* scales, void* biases,
                            cudaStream_t st) {
  if (w_dtype == QMM_F32)
    return launch_quant_s<float>(s_dtype, bits, w, rows, cols, gs, packed, scales, biases, st);
  if (w_dtype == QMM_BF16)
    return launch_quant_s<__nv_bfloat16>(s_dtype, bits, w, rows, cols, gs, packed, scales, biases, st);
  return launch_quant_s<__half>(s_dtype, bits, w, rows, cols, gs, packed, scales, biases, st);
}

template <int B, typename TS>
static cudaError_t launch_deq_o(int out_dtype, const qmm_qweight* w, void* out, cudaStream_t st) {
  const int64_t n = w->rows * (w->cols / 32);
  const int blocks = (int)((n + 255) / 256);
  auto S = reinterpret_cast<const TS*>(w->scales);
  auto Bi = reinterpret_cast<const TS*>(w->biases);
  if (out_dtype == QMM_F32)
    dequant_kernel<B, TS, float><<<blocks, 256, 0, st>>>(w->packed, S, Bi, w->rows, w->cols,
                                                          w->group_size, (float*)out);
  else if (out_dtype == QMM_BF16)
    dequant_kernel<B, TS, __nv_bfloat16><<<blocks, 256, 0, st>>>(
        w->packed, S, Bi, w->rows, w->cols, w->group_size, (__nv_bfloat16*)out);
  else
    dequant_kernel<B, TS, __half><<<blocks, 256, 0, st>>>(w->packed, S, Bi, w->rows, w->cols,
                                                           w->group_size, (__half*)out);
  return cudaGetLastError();
}

template <typename TS>
static cudaError_t launch_deq_b(int out_dtype, const qmm_qweight* w, void* out, cudaStream_t st) {
  switch (w->bits) {
    case 2: return launch_deq_o<2, TS>(out_dtype, w, out, st);
    case 3: return launch_deq_o<3, TS>(out_dtype, w, out, st);
    case 4: return launch_deq_o<4, TS>(out_dtype, w, out, st);
    case 6: return launch_deq_o<6, TS>(out_dtype, w, out, st);
    default: return launch_deq_o<8, TS>(out_dtype, w, out, st);
  }
}

cudaError_t launch_dequantize(const qmm_qweight* w, void* out, int out_dtype, cudaStream_t st) {
  if (w->sdtype == QMM_F32) return launch_deq_b<float>(out_dtype, w, out, st);
  if (w->sdtype == QMM_BF16) return launch_deq_b<__nv_bfloat16>(out_dtype, w, out, st);
  return launch_deq_b<__half>(out_dtype, w, out, st);
}

}  // namespace qmm
