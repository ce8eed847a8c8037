// Microscaled modes ("emily 0.5.1 lib/emily/quantization.ex",
// dequantize_mxfp4_impl, dequantize_mxfp8_impl, dequantize_nvfp4_impl):
//   mxfp4: 4-bit FP4-E2M1 lanes, one FP8-E8M0 scale byte per 32 lanes
//   mxfp8: 8-bit FP8-E4M3 lanes, one FP8-E8M0 scale byte per 32 lanes
//   nvfp4: 4-bit FP4-E2M1 lanes, one FP8-E4M3 scale byte per 16 lanes
//   w_hat = lane(q) * scale(s), no bias; lanes LSB-first in u32 words.
// E8M0 is 2^(s - 127).  FP8-E4M3 is decoded the way the page does it: the
// low 7 bits shifted left by 7 read as a binary16, times 256, with the sign
// of bit 7 (so 0x7F / 0xFF are +-480, not NaN).
//
// Kernels: the standalone dequantization (bit-exact: one fp32 product, one
// rounding to the output dtype) and a CUDA-core matmul for these modes
// (fp32 products and sums; one warp per weight row, the lanes splitting K in
// 32-code chunks, up to 8 tokens per pass).
#include <algorithm>

#include "common.cuh"

namespace qmm {
namespace mx {

__device__ __forceinline__ float e2m1(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  // e = 0: subnormal 0.5 m; else 2^(e - 1) (1 + m / 2)
  const float mag = e == 0 ? 0.5f * (float)m : __int_as_float((int)(e + 126u) << 23) * (1.0f + 0.5f * (float)m);
  return (c & 8u) ? -mag : mag;
}
__device__ __forceinline__ float e8m0(uint32_t s) {
  s &= 0xffu;
  // exponent field s with a zero fraction is 2^(s - 127); s = 0 is 2^-127
  // (a subnormal), s = 255 reads as +inf
  return s == 0 ? __int_as_float(0x00400000) : __int_as_float((int)(s << 23));
}
__device__ __forceinline__ float e4m3(uint32_t b) {
  const float mag = __half2float(__ushort_as_half((unsigned short)((b & 0x7fu) << 7))) * 256.0f;
  return (b & 0x80u) ? -mag : mag;
}

template <int MODE>
struct Mode;
template <>
struct Mode<QMM_MODE_MXFP4> {
  static constexpr int B = 4, GS = 32;
  __device__ static float lane(uint32_t c) { return e2m1(c); }
  __device__ static float scale(uint32_t s) { return e8m0(s); }
};
template <>
struct Mode<QMM_MODE_MXFP8> {
  static constexpr int B = 8, GS = 32;
  __device__ static float lane(uint32_t c) { return e4m3(c); }
  __device__ static float scale(uint32_t s) { return e8m0(s); }
};
template <>
struct Mode<QMM_MODE_NVFP4> {
  static constexpr int B = 4, GS = 16;
  __device__ static float lane(uint32_t c) { return e2m1(c); }
  __device__ static float scale(uint32_t s) { return e4m3(s); }
};

// One thread per 32 consecutive lanes of a row (B whole words).
template <int MODE, typename TO>
__global__ void __launch_bounds__(256)
dequant_mx_kernel(const uint32_t* __restrict__ packed, const uint8_t* __restrict__ scales, int64_t rows,
                  int64_t cols, TO* __restrict__ out) {
  using Md = Mode<MODE>;
  constexpr int B = Md::B, GS = Md::GS;
  const int64_t chunks = cols / 32;
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (idx >= rows * chunks) return;
  const int64_t r = idx / chunks, c = idx % chunks;
  const int64_t G = cols / GS;
  const uint32_t* src = packed + r * (cols * B / 32) + c * B;
  uint32_t wr[B];
#pragma unroll
  for (int i = 0; i < B; ++i) wr[i] = __ldg(src + i);
  TO vals[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t q = (wr[(i * B) >> 5] >> ((i * B) & 31)) & ((1u << B) - 1u);
    const float s = Md::scale(__ldg(scales + r * G + (c * 32 + i) / GS));
    vals[i] = from_f32<TO>(Md::lane(q) * s);
  }
  uint4* dst = reinterpret_cast<uint4*>(out + r * cols + c * 32);
  const uint4* v4 = reinterpret_cast<const uint4*>(vals);
#pragma unroll
  for (int i = 0; i < (int)(32 * sizeof(TO) / 16); ++i) dst[i] = v4[i];
}

constexpr int kMB = 8;  // tokens per pass

// y[m, n] = sum_k x[m, k] w_hat[n, k]: one warp per row n (grid-stride), lane
// l takes the 32-lane chunks l, l + 32, ... of the row.
template <int MODE, typename TX>
__global__ void __launch_bounds__(256)
matmul_mx_kernel(const TX* __restrict__ x, int64_t M, int64_t K, const uint32_t* __restrict__ packed,
                 const uint8_t* __restrict__ scales, int64_t N, void* y, int64_t ldy, int y_dtype) {
  using Md = Mode<MODE>;
  constexpr int B = Md::B, GS = Md::GS;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  const int64_t chunks = K / 32, wpr = K * B / 32, G = K / GS;
  for (int64_t n = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5); n < N; n += warps) {
    const uint32_t* row = packed + n * wpr;
    for (int64_t m0 = 0; m0 < M; m0 += kMB) {
      float acc[kMB];
#pragma unroll
      for (int i = 0; i < kMB; ++i) acc[i] = 0.0f;
      for (int64_t c = lane; c < chunks; c += 32) {
        uint32_t wr[B];
#pragma unroll
        for (int i = 0; i < B; ++i) wr[i] = __ldg(row + c * B + i);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint32_t q = (wr[(i * B) >> 5] >> ((i * B) & 31)) & ((1u << B) - 1u);
          const int64_t k = c * 32 + i;
          const float w = Md::lane(q) * Md::scale(__ldg(scales + n * G + k / GS));
#pragma unroll
          for (int t = 0; t < kMB; ++t)
            if (m0 + t < M) acc[t] = fmaf(to_f32(x[(m0 + t) * K + k]), w, acc[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < kMB; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
      }
      if (lane == 0)
        for (int t = 0; t < kMB; ++t)
          if (m0 + t < M) store_as(y, y_dtype, (m0 + t) * ldy + n, acc[t]);
    }
  }
}

template <int MODE>
static cudaError_t dequant_m(const qmm_qweight* w, void* out, int out_dtype, cudaStream_t st) {
  const int64_t n = w->rows * (w->cols / 32);
  const int blocks = (int)((n + 255) / 256);
  auto S = reinterpret_cast<const uint8_t*>(w->scales);
  if (out_dtype == QMM_F32)
    dequant_mx_kernel<MODE, float><<<blocks, 256, 0, st>>>(w->packed, S, w->rows, w->cols, (float*)out);
  else if (out_dtype == QMM_BF16)
    dequant_mx_kernel<MODE, __nv_bfloat16><<<blocks, 256, 0, st>>>(w->packed, S, w->rows, w->cols,
                                                                  (__nv_bfloat16*)out);
  else
    dequant_mx_kernel<MODE, __half><<<blocks, 256, 0, st>>>(w->packed, S, w->rows, w->cols, (__half*)out);
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t matmul_m(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w, void* y,
                            int64_t ldy, int y_dtype, cudaStream_t st) {
  auto S = reinterpret_cast<const uint8_t*>(w->scales);
  const int64_t N = w->rows;
  const int blocks = (int)std::min<int64_t>((N + 7) / 8, 148 * 8);
  if (x_dtype == QMM_F32)
    matmul_mx_kernel<MODE, float><<<blocks, 256, 0, st>>>((const float*)x, M, K, w->packed, S, N, y, ldy, y_dtype);
  else if (x_dtype == QMM_BF16)
    matmul_mx_kernel<MODE, __nv_bfloat16><<<blocks, 256, 0, st>>>((const __nv_bfloat16*)x, M, K, w->packed, S,
                                                                  N, y, ldy, y_dtype);
  else
    matmul_mx_kernel<MODE, __half><<<blocks, 256, 0, st>>>((const __half*)x, M, K, w->packed, S, N, y, ldy, y_dtype);
  return cudaGetLastError();
}

}  // namespace mx

cudaError_t launch_dequantize_mx(const qmm_qweight* w, void* out, int out_dtype, cudaStream_t st) {
  switch (w->mode) {
    case QMM_MODE_MXFP4: return mx::dequant_m<QMM_MODE_MXFP4>(w, out, out_dtype, st);
    case QMM_MODE_MXFP8: return mx::dequant_m<QMM_MODE_MXFP8>(w, out, out_dtype, st);
    default: return mx::dequant_m<QMM_MODE_NVFP4>(w, out, out_dtype, st);
  }
}

cudaError_t launch_matmul_mx(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w, void* y,
                             int64_t ldy, int y_dtype, cudaStream_t st) {
  switch (w->mode) {
    case QMM_MODE_MXFP4: return mx::matmul_m<QMM_MODE_MXFP4>(x, x_dtype, M, K, w, y, ldy, y_dtype, st);
    case QMM_MODE_MXFP8: return mx::matmul_m<QMM_MODE_MXFP8>(x, x_dtype, M, K, w, y, ldy, y_dtype, st);
    default: return mx::matmul_m<QMM_MODE_NVFP4>(x, x_dtype, M, K, w, y, ldy, y_dtype, st);
  }
}

}  // namespace qmm
