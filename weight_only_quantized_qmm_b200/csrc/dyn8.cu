// Per-tensor dynamic-range int8 ("mlex 0.1.3 src/quant.rs",
// DynamicRangeParams, quantize_dynamic_int8, dequantize_dynamic_int8):
//   params = {input_min, input_max, output_min, output_max}
//   w_hat  = fl(fl(fl(q + 128) * scale) + output_min),
//   scale  = fl((output_max - output_min) / 255)
// and the quantizer that writes such a tensor from its own min and max:
//   scale = max((max - min) / 255, FLT_EPSILON),
//   q = clamp(round((w - min) / scale) - 128, -128, 127), NaN -> 0,
// with the min/max fold passing over NaN elements.
//
// Kernels:
//   * quantize: an ordered-integer min/max reduction (one atomicMin/Max per
//     block into the params buffer), the code pass, and a one-thread pass
//     that writes the four float params; all fp32 steps bit-exact (_rn
//     intrinsics, nothing contracted);
//   * dequantize: 16 codes per thread, the page's three roundings;
//   * matmul y = x . w_hat^T (W is [N, K] int8): one warp per weight row,
//     16 codes per lane per step, x staged in shared memory as fp32 for up to
//     8 tokens per pass.  Each code becomes u = q + 128 exactly (the byte
//     with its top bit flipped, placed under the exponent of 2^23 by one
//     prmt), and a row's dot is regrouped as
//       y = scale * sum_k x_k u_k + output_min * sum_k x_k,
//     the same sum as sum_k x_k w_hat_k but for the per-element rounding of
//     w_hat (fp32 accumulation either way).
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace qmm {
namespace dyn8 {

// int32 key with the order of the float (for atomicMin / atomicMax)
__device__ __forceinline__ int key_of(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float float_of(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }

// params[0], params[1] hold the min / max keys until the last pass
__global__ void init_kernel(float* params) {
  reinterpret_cast<int*>(params)[0] = key_of(INFINITY);
  reinterpret_cast<int*>(params)[1] = key_of(-INFINITY);
}

template <typename T>
__global__ void __launch_bounds__(256) minmax_kernel(const T* __restrict__ w, int64_t n, float* params) {
  float mn = INFINITY, mx = -INFINITY;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float v = to_f32(w[i]);
    mn = fminf(mn, v);  // fminf / fmaxf pass over NaN
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  __shared__ float smn[8], smx[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { smn[warp] = mn; smx[warp] = mx; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) { mn = fminf(mn, smn[i]); mx = fmaxf(mx, smx[i]); }
    atomicMin(reinterpret_cast<int*>(params), key_of(mn));
    atomicMax(reinterpret_cast<int*>(params) + 1, key_of(mx));
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
quant_kernel(const T* __restrict__ w, int64_t n, const float* __restrict__ params, int8_t* __restrict__ q) {
  const float mn = float_of(reinterpret_cast<const int*>(params)[0]);
  const float mx = float_of(reinterpret_cast<const int*>(params)[1]);
  float scale = __fdiv_rn(__fsub_rn(mx, mn), 255.0f);
  if (!(scale >= FLT_EPSILON)) scale = FLT_EPSILON;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float t = __fsub_rn(roundf(__fdiv_rn(__fsub_rn(to_f32(w[i]), mn), scale)), 128.0f);
    q[i] = t != t ? (int8_t)0 : (int8_t)(int)fminf(fmaxf(t, -128.0f), 127.0f);
  }
}

__global__ void finalize_kernel(float* params) {
  const float mn = float_of(reinterpret_cast<const int*>(params)[0]);
  const float mx = float_of(reinterpret_cast<const int*>(params)[1]);
  params[0] = mn;
  params[1] = mx;
  params[2] = mn;
  params[3] = mx;
}

__device__ __forceinline__ float w_hat(int q, float scale, float omin) {
  return __fadd_rn(__fmul_rn(__fadd_rn((float)q, 128.0f), scale), omin);
}

// 16 codes per thread; the last partial chunk one code at a time
template <typename TO>
__global__ void __launch_bounds__(256)
dequant_kernel(const int8_t* __restrict__ q, int64_t n, const float* __restrict__ params, TO* __restrict__ out) {
  const float scale = __fdiv_rn(__fsub_rn(params[3], params[2]), 255.0f), omin = params[2];
  const int64_t chunks = n / 16;
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c <= chunks; c += (int64_t)gridDim.x * blockDim.x) {
    if (c < chunks) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(q) + c);
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
      __align__(16) TO o[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) o[i] = from_f32<TO>(w_hat((int)(int8_t)(wv[i >> 2] >> (8 * (i & 3))), scale, omin));
      uint4* dst = reinterpret_cast<uint4*>(out + c * 16);
#pragma unroll
      for (int i = 0; i < (int)(16 * sizeof(TO) / 16); ++i) dst[i] = reinterpret_cast<const uint4*>(o)[i];
    } else {
      for (int64_t i = chunks * 16; i < n; ++i) out[i] = from_f32<TO>(w_hat(q[i], scale, omin));
    }
  }
}

constexpr int kTok = 8;    // tokens per pass
constexpr int kBatch = 8;  // 16-byte weight chunks a lane requests at once

// 16 bytes read once: not kept in L1
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// byte j of w (already XOR-ed with 0x80) as a float: 2^23 + u, minus 2^23
template <int J>
__device__ __forceinline__ float byte_u(uint32_t w) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(0x4Bu), "n"(0x4550 | J));
  return __int_as_float((int)r) - 8388608.0f;
}

// One warp per weight row; XS: x staged in shared memory (else read from
// global memory, for rows too long to stage).  VEC: K % 16 == 0 and 16-byte
// aligned rows.
template <typename TX, bool XS, bool VEC>
__global__ void __launch_bounds__(256)
matmul_kernel(const TX* __restrict__ x, int64_t M, int64_t K, const int8_t* __restrict__ q, int64_t N,
              const float* __restrict__ params, void* y, int y_dtype) {
  extern __shared__ float xs[];  // [kTok][K] when XS
  __shared__ float xsum[kTok];
  __shared__ float wpart[8];
  const float scale = __fdiv_rn(__fsub_rn(params[3], params[2]), 255.0f), omin = params[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t m0 = 0; m0 < M; m0 += kTok) {
    const int mb = (int)(M - m0 < kTok ? M - m0 : kTok);
    __syncthreads();  // the previous pass is done with xs
    for (int t = 0; t < mb; ++t) {
      // sum of x in a fixed order (thread, then warp, then block)
      float s = 0.0f;
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
        const float v = to_f32(x[(m0 + t) * K + k]);
        if (XS) xs[t * K + k] = v;
        s += v;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) wpart[warp] = s;
      __syncthreads();
      if (threadIdx.x == 0) {
        float b = 0.0f;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) b += wpart[i];
        xsum[t] = b;
      }
      __syncthreads();
    }
    for (int64_t n = blockIdx.x * (int64_t)(blockDim.x >> 5) + warp; n < N; n += warps) {
      float acc[kTok];
#pragma unroll
      for (int t = 0; t < kTok; ++t) acc[t] = 0.0f;
      const int8_t* row = q + n * K;
      if (VEC) {
        // kBatch 16-byte chunks per lane are requested before any of them is
        // used, so that a warp keeps up to kBatch * 512 bytes of its row in
        // flight
        const int64_t nch = K / 16;
        for (int64_t cb = 0; cb < nch; cb += 32 * kBatch) {
          uint4 vb[kBatch];
#pragma unroll
          for (int j = 0; j < kBatch; ++j) {
            const int64_t c = cb + lane + 32 * j;
            vb[j] = c < nch ? ld_stream(reinterpret_cast<const uint4*>(row) + c) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int jb = 0; jb < kBatch; ++jb) {
          const int64_t c = cb + lane + 32 * jb;
          if (c < nch) {
          const uint4 v = vb[jb];
          const uint32_t wv[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u, v.w ^ 0x80808080u};
          float u[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            u[4 * j] = byte_u<0>(wv[j]);
            u[4 * j + 1] = byte_u<1>(wv[j]);
            u[4 * j + 2] = byte_u<2>(wv[j]);
            u[4 * j + 3] = byte_u<3>(wv[j]);
          }
#pragma unroll
          for (int t = 0; t < kTok; ++t) {
            if (t < mb) {
              const int64_t k0 = c * 16;
#pragma unroll
              for (int j = 0; j < 16; j += 4) {
                float4 xv;
                if (XS) {
                  xv = *reinterpret_cast<const float4*>(xs + t * K + k0 + j);
                } else {
                  const TX* xp = x + (m0 + t) * K + k0 + j;
                  xv = make_float4(to_f32(xp[0]), to_f32(xp[1]), to_f32(xp[2]), to_f32(xp[3]));
                }
                acc[t] = fmaf(xv.x, u[j], acc[t]);
                acc[t] = fmaf(xv.y, u[j + 1], acc[t]);
                acc[t] = fmaf(xv.z, u[j + 2], acc[t]);
                acc[t] = fmaf(xv.w, u[j + 3], acc[t]);
              }
            }
          }
          }
          }
        }
      } else {
        for (int64_t k = lane; k < K; k += 32) {
          const float u = (float)((int)row[k] + 128);
#pragma unroll
          for (int t = 0; t < kTok; ++t)
            if (t < mb) acc[t] = fmaf(XS ? xs[t * K + k] : to_f32(x[(m0 + t) * K + k]), u, acc[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < kTok; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
      }
      if (lane == 0)
        for (int t = 0; t < mb; ++t) store_as(y, y_dtype, (m0 + t) * N + n, fmaf(scale, acc[t], omin * xsum[t]));
    }
  }
}

template <typename T>
cudaError_t quantize_t(const T* w, int64_t n, int8_t* q, float* params, cudaStream_t st) {
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)qmm_host::num_sms() * 8);
  init_kernel<<<1, 1, 0, st>>>(params);
  minmax_kernel<T><<<blocks, 256, 0, st>>>(w, n, params);
  quant_kernel<T><<<blocks, 256, 0, st>>>(w, n, params, q);
  finalize_kernel<<<1, 1, 0, st>>>(params);
  return cudaGetLastError();
}

template <typename TO>
cudaError_t dequant_t(const int8_t* q, int64_t n, const float* params, TO* out, cudaStream_t st) {
  const int64_t threads = n / 16 + 1;
  const int blocks = (int)std::min<int64_t>((threads + 255) / 256, (int64_t)qmm_host::num_sms() * 16);
  dequant_kernel<TO><<<blocks, 256, 0, st>>>(q, n, params, out);
  return cudaGetLastError();
}

constexpr int64_t kXsMax = 160 * 1024;  // shared-memory bytes for staged x

template <typename TX, bool XS, bool VEC>
cudaError_t matmul_v(const TX* x, int64_t M, int64_t K, const int8_t* q, int64_t N, const float* params, void* y,
                     int y_dtype, cudaStream_t st) {
  auto k = matmul_kernel<TX, XS, VEC>;
  const size_t smem = XS ? (size_t)std::min<int64_t>(M, kTok) * K * 4 : 0;
  if (XS) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kXsMax);
    if (e != cudaSuccess) return e;
  }
  const int blocks = (int)std::min<int64_t>((N + 7) / 8, (int64_t)qmm_host::num_sms() * (smem > 100 * 1024 ? 1 : 2));
  k<<<blocks, 256, smem, st>>>(x, M, K, q, N, params, y, y_dtype);
  return cudaGetLastError();
}

template <typename TX>
cudaError_t matmul_t(const TX* x, int64_t M, int64_t K, const int8_t* q, int64_t N, const float* params, void* y,
                     int y_dtype, cudaStream_t st) {
  const bool xs = std::min<int64_t>(M, kTok) * K * 4 <= kXsMax;
  const bool vec = K % 16 == 0;  // q is 16-byte aligned (checked by the caller)
  if (xs && vec) return matmul_v<TX, true, true>(x, M, K, q, N, params, y, y_dtype, st);
  if (xs) return matmul_v<TX, true, false>(x, M, K, q, N, params, y, y_dtype, st);
  if (vec) return matmul_v<TX, false, true>(x, M, K, q, N, params, y, y_dtype, st);
  return matmul_v<TX, false, false>(x, M, K, q, N, params, y, y_dtype, st);
}

}  // namespace dyn8

cudaError_t launch_quantize_dyn8(const void* w, int w_dtype, int64_t n, int8_t* q, float* params, cudaStream_t st) {
  if (w_dtype == QMM_F32) return dyn8::quantize_t((const float*)w, n, q, params, st);
  if (w_dtype == QMM_BF16) return dyn8::quantize_t((const __nv_bfloat16*)w, n, q, params, st);
  return dyn8::quantize_t((const __half*)w, n, q, params, st);
}

cudaError_t launch_dequantize_dyn8(const int8_t* q, int64_t n, const float* params, void* out, int out_dtype,
                                   cudaStream_t st) {
  if (out_dtype == QMM_F32) return dyn8::dequant_t(q, n, params, (float*)out, st);
  if (out_dtype == QMM_BF16) return dyn8::dequant_t(q, n, params, (__nv_bfloat16*)out, st);
  return dyn8::dequant_t(q, n, params, (__half*)out, st);
}

cudaError_t launch_matmul_dyn8(const void* x, int x_dtype, int64_t M, int64_t K, const int8_t* q, int64_t N,
                               const float* params, void* y, int y_dtype, cudaStream_t st) {
  if (x_dtype == QMM_F32) return dyn8::matmul_t((const float*)x, M, K, q, N, params, y, y_dtype, st);
  if (x_dtype == QMM_BF16) return dyn8::matmul_t((const __nv_bfloat16*)x, M, K, q, N, params, y, y_dtype, st);
  return dyn8::matmul_t((const __half*)x, M, K, q, N, params, y, y_dtype, st);
}

}  // namespace qmm
