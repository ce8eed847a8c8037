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
// 32-code chunks requested several at a time, each lane decoded by shifts
// into an exact f16, the group scale applied once per group partial; up to 8
// tokens per pass).
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

constexpr int kMB = 8;      // tokens per pass
constexpr int kBatch = 4;   // 32-code chunks a lane requests at once
constexpr int64_t kXsMax = 128 * 1024;  // shared-memory bytes for staged x

// Lanes of one packed word as exact f16 pairs, scaled by a power of two that
// the group scale takes back:
//   E2M1 (4-bit): the code's exponent and mantissa bits under bits 9..11 of
//     an f16 read as 2^-14 * lane (the exponent bias 15 against E2M1's 1; a
//     zero exponent field gives the f16 subnormal 2^-15 m, which is
//     2^-14 * 0.5 m); pair j = codes j and j + 4;
//   E4M3 (8-bit, the page's decode): the low 7 bits under bits 7..13 of an
//     f16 read as lane / 256; pair j = codes j and j + 2.
template <int B>
__device__ __forceinline__ void lanes_f32(uint32_t w, float* v) {
  if constexpr (B == 4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t x = w >> (4 * j);
      const uint32_t h = ((x << 9) & 0x0E000E00u) | ((x << 12) & 0x80008000u);
      __half2 hh;
      memcpy(&hh, &h, 4);
      const float2 f = __half22float2(hh);
      v[j] = f.x;
      v[j + 4] = f.y;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t x = w >> (8 * j);
      const uint32_t h = ((x & 0x007F007Fu) << 7) | ((x & 0x00800080u) << 8);
      __half2 hh;
      memcpy(&hh, &h, 4);
      const float2 f = __half22float2(hh);
      v[j] = f.x;
      v[j + 2] = f.y;
    }
  }
}

// y[m, n] = sum_k x[m, k] w_hat[n, k]: one warp per row n (grid-stride); lane
// l takes the 32-code chunks l, l + 32, ..., kBatch of them per request; per
// group the partial dot sum_k x_k lane_k is taken first and then scaled.
// XS: x staged in shared memory as fp32, each 32-value chunk padded to 36
// floats so that the lanes' 16-byte reads of their chunks (144 bytes apart)
// fall in distinct banks.  MB: tokens per pass (1 for a single
// token, so that no predicated-off token work is issued; else kMB).
template <int MODE, typename TX, bool XS, int MB>
__global__ void __launch_bounds__(256)
matmul_mx_kernel(const TX* __restrict__ x, int64_t M, int64_t K, const uint32_t* __restrict__ packed,
                 const uint8_t* __restrict__ scales, int64_t N, void* y, int64_t ldy, int y_dtype) {
  constexpr int kMB = MB;
  using Md = Mode<MODE>;
  constexpr int B = Md::B, GS = Md::GS, GPC = 32 / GS;  // groups per 32-code chunk
  constexpr float kLaneUnit = B == 4 ? 16384.0f : 256.0f;
  extern __shared__ float xs[];  // [kMB][K / 32][36] when XS
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  const int64_t chunks = K / 32, wpr = K * B / 32, G = K / GS;
  const int64_t KP = chunks * 36;  // padded staged row
  for (int64_t m0 = 0; m0 < M; m0 += kMB) {
    const int mb = (int)(M - m0 < kMB ? M - m0 : kMB);
    if (XS) {
      __syncthreads();
      for (int64_t i = threadIdx.x; i < (int64_t)mb * K; i += blockDim.x) {
        const int64_t t = i / K, k = i - t * K;
        xs[t * KP + (k >> 5) * 36 + (k & 31)] = to_f32(x[m0 * K + i]);
      }
      __syncthreads();
    }
    for (int64_t n = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5); n < N; n += warps) {
      const uint32_t* row = packed + n * wpr;
      float acc[kMB];
#pragma unroll
      for (int t = 0; t < kMB; ++t) acc[t] = 0.0f;
      for (int64_t cb = 0; cb < chunks; cb += 32 * kBatch) {
        uint32_t wv[kBatch][B];
        uint32_t sb[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const int64_t c = cb + lane + 32 * j;
          const int64_t cc = c < chunks ? c : 0;
#pragma unroll
          for (int q = 0; q < B / 4; ++q) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + cc * B) + q);
            wv[j][4 * q] = v.x; wv[j][4 * q + 1] = v.y; wv[j][4 * q + 2] = v.z; wv[j][4 * q + 3] = v.w;
          }
          sb[j] = GPC == 1 ? (uint32_t)__ldg(scales + n * G + cc)
                           : (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(scales + n * G) + cc);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const int64_t c = cb + lane + 32 * j;
          if (c < chunks) {
            float lv[32];
#pragma unroll
            for (int q = 0; q < B; ++q) lanes_f32<B>(wv[j][q], lv + q * (32 / B));
            float sc[GPC];
#pragma unroll
            for (int gi = 0; gi < GPC; ++gi) sc[gi] = Md::scale(sb[j] >> (8 * gi)) * kLaneUnit;
#pragma unroll
            for (int t = 0; t < kMB; ++t) {
              if (t < mb) {
#pragma unroll
                for (int gi = 0; gi < GPC; ++gi) {
                  float part = 0.0f;
#pragma unroll
                  for (int i = gi * GS; i < (gi + 1) * GS; i += 4) {
                    float4 xv;
                    if (XS) {
                      xv = *reinterpret_cast<const float4*>(xs + t * KP + c * 36 + i);
                    } else {
                      const TX* xp = x + (m0 + t) * K + c * 32 + i;
                      xv = make_float4(to_f32(xp[0]), to_f32(xp[1]), to_f32(xp[2]), to_f32(xp[3]));
                    }
                    part = fmaf(xv.x, lv[i], part);
                    part = fmaf(xv.y, lv[i + 1], part);
                    part = fmaf(xv.z, lv[i + 2], part);
                    part = fmaf(xv.w, lv[i + 3], part);
                  }
                  acc[t] = fmaf(sc[gi], part, acc[t]);
                }
              }
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kMB; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
      }
      if (lane == 0)
        for (int t = 0; t < mb; ++t) store_as(y, y_dtype, (m0 + t) * ldy + n, acc[t]);
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

template <int MODE, typename TX>
static cudaError_t matmul_x(const TX* x, int64_t M, int64_t K, const qmm_qweight* w, void* y, int64_t ldy,
                            int y_dtype, cudaStream_t st) {
  auto S = reinterpret_cast<const uint8_t*>(w->scales);
  const int64_t N = w->rows;
  const int64_t row_bytes = (K / 32) * 36 * 4;  // a staged (padded) row of x
  const bool xs = (M < kMB ? M : kMB) * row_bytes <= kXsMax;
  const size_t smem = xs ? (size_t)(M < kMB ? M : kMB) * row_bytes : 0;
  auto k = xs ? (M == 1 ? matmul_mx_kernel<MODE, TX, true, 1> : matmul_mx_kernel<MODE, TX, true, kMB>)
              : (M == 1 ? matmul_mx_kernel<MODE, TX, false, 1> : matmul_mx_kernel<MODE, TX, false, kMB>);
  if (xs) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kXsMax);
    if (e != cudaSuccess) return e;
  }
  // as many resident blocks per SM as registers and the staged x allow (at
  // most 4): more rows' loads in flight (measured, one token, 14336 x 4096:
  // -2 to -5% against two blocks per SM); one wave, so that the grid-stride
  // row loop has no tail of late blocks
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 256, smem) != cudaSuccess || per_sm < 1) per_sm = 1;
  const int blocks = (int)std::min<int64_t>((N + 7) / 8, (int64_t)qmm_host::num_sms() * std::min(per_sm, 4));
  k<<<blocks, 256, smem, st>>>(x, M, K, w->packed, S, N, y, ldy, y_dtype);
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t matmul_m(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w, void* y,
                            int64_t ldy, int y_dtype, cudaStream_t st) {
  if (x_dtype == QMM_F32) return matmul_x<MODE>((const float*)x, M, K, w, y, ldy, y_dtype, st);
  if (x_dtype == QMM_BF16) return matmul_x<MODE>((const __nv_bfloat16*)x, M, K, w, y, ldy, y_dtype, st);
  return matmul_x<MODE>((const __half*)x, M, K, w, y, ldy, y_dtype, st);
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
