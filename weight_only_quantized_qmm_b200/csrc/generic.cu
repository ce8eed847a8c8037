// CUDA-core quantized matmul for the cases the tensor-core kernels do not
// take: fp32 activations, the transposed (AWQ) layout, and any M for them.
// Correctness path: w_hat = fmaf(q, s, b) in fp32 per element, fp32 sums.
//
// transpose = 1: y[m, n] = sum_k x[m, k] w_hat[n, k]   (W is [N, K])
// transpose = 0: y[m, n] = sum_k x[m, k] w_hat[k, n]   (W is [K, N], quantized
//                along N: "emily 0.5.1 lib/emily/quantization.ex",
//                quantized_matmul/2, the AWQ convention when transpose is false)
#include "common.cuh"

namespace qmm {

constexpr int kMB = 8;  // tokens per pass

template <int B>
__device__ __forceinline__ uint32_t code_of(const uint32_t* row, int64_t i) {
  const int64_t bit = i * B;
  const int64_t w = bit >> 5;
  const int sh = (int)(bit & 31);
  uint32_t v = row[w] >> sh;
  if (sh + B > 32) v |= row[w + 1] << (32 - sh);
  return v & ((1u << B) - 1u);
}

// one warp per output column n; lanes split K; kMB tokens per pass
template <int B, typename TX>
__global__ void __launch_bounds__(256)
generic_t1_kernel(const TX* __restrict__ x, int64_t M, int64_t K, const uint32_t* __restrict__ packed,
                  const TX* __restrict__ scales, const TX* __restrict__ biases, int64_t N, int gs,
                  void* y, int64_t ldy, int y_dtype) {
  const int lane = threadIdx.x & 31;
  const int64_t n = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5);
  if (n >= N) return;
  const int64_t wpr = K * B / 32, G = K / gs;
  const uint32_t* row = packed + n * wpr;
  for (int64_t m0 = 0; m0 < M; m0 += kMB) {
    float acc[kMB];
#pragma unroll
    for (int i = 0; i < kMB; ++i) acc[i] = 0.0f;
    for (int64_t k = lane; k < K; k += 32) {
      const int64_t g = k / gs;
      const float w = fmaf((float)code_of<B>(row, k), to_f32(scales[n * G + g]), to_f32(biases[n * G + g]));
#pragma unroll
      for (int i = 0; i < kMB; ++i)
        if (m0 + i < M) acc[i] = fmaf(to_f32(x[(m0 + i) * K + k]), w, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < kMB; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    }
    if (lane == 0)
      for (int i = 0; i < kMB; ++i)
        if (m0 + i < M) store_as(y, y_dtype, (m0 + i) * ldy + n, acc[i]);
  }
}

// one thread per (token block, output column n); walks K
template <int B, typename TX>
__global__ void __launch_bounds__(256)
generic_t0_kernel(const TX* __restrict__ x, int64_t M, int64_t K, const uint32_t* __restrict__ packed,
                  const TX* __restrict__ scales, const TX* __restrict__ biases, int64_t N, int gs,
                  void* y, int64_t ldy, int y_dtype) {
  const int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t m0 = (int64_t)blockIdx.y * kMB;
  if (n >= N) return;
  const int64_t wpr = N * B / 32, G = N / gs;
  float acc[kMB];
#pragma unroll
  for (int i = 0; i < kMB; ++i) acc[i] = 0.0f;
  for (int64_t k = 0; k < K; ++k) {
    const uint32_t* row = packed + k * wpr;
    const float w = fmaf((float)code_of<B>(row, n), to_f32(scales[k * G + n / gs]), to_f32(biases[k * G + n / gs]));
#pragma unroll
    for (int i = 0; i < kMB; ++i)
      if (m0 + i < M) acc[i] = fmaf(to_f32(x[(m0 + i) * K + k]), w, acc[i]);
  }
  for (int i = 0; i < kMB; ++i)
    if (m0 + i < M) store_as(y, y_dtype, (m0 + i) * ldy + n, acc[i]);
}

template <int B, typename TX>
static cudaError_t launch_g(const void* x, int64_t M, int64_t K, const qmm_qweight* w,
                            int transpose, void* y, int64_t ldy, int y_dtype, cudaStream_t st) {
  auto X = reinterpret_cast<const TX*>(x);
  auto S = reinterpret_cast<const TX*>(w->scales);
  auto Bi = reinterpret_cast<const TX*>(w->biases);
  if (transpose) {
    const int64_t N = w->rows;
    const int blocks = (int)((N + 7) / 8);
    generic_t1_kernel<B, TX><<<blocks, 256, 0, st>>>(X, M, K, w->packed, S, Bi, N, w->group_size, y, ldy, y_dtype);
  } else {
    const int64_t N = w->cols;
    dim3 grid((unsigned)((N + 255) / 256), (unsigned)((M + kMB - 1) / kMB));
    generic_t0_kernel<B, TX><<<grid, 256, 0, st>>>(X, M, K, w->packed, S, Bi, N, w->group_size, y, ldy, y_dtype);
  }
  return cudaGetLastError();
}

template <typename TX>
static cudaError_t launch_gb(const void* x, int64_t M, int64_t K, const qmm_qweight* w,
                             int transpose, void* y, int64_t ldy, int y_dtype, cudaStream_t st) {
  switch (w->bits) {
    case 2: return launch_g<2, TX>(x, M, K, w, transpose, y, ldy, y_dtype, st);
    case 3: return launch_g<3, TX>(x, M, K, w, transpose, y, ldy, y_dtype, st);
    case 4: return launch_g<4, TX>(x, M, K, w, transpose, y, ldy, y_dtype, st);
    case 6: return launch_g<6, TX>(x, M, K, w, transpose, y, ldy, y_dtype, st);
    default: return launch_g<8, TX>(x, M, K, w, transpose, y, ldy, y_dtype, st);
  }
}

cudaError_t launch_generic(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w,
                           int transpose, void* y, int64_t ldy, int y_dtype, cudaStream_t st) {
  if (x_dtype == QMM_F32) return launch_gb<float>(x, M, K, w, transpose, y, ldy, y_dtype, st);
  if (x_dtype == QMM_BF16) return launch_gb<__nv_bfloat16>(x, M, K, w, transpose, y, ldy, y_dtype, st);
  return launch_gb<__half>(x, M, K, w, transpose, y, ldy, y_dtype, st);
}

}  // namespace qmm
