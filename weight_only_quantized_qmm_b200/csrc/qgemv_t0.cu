// Quantized matmul with the weight stored [K, N] and quantized along N
// ("emily 0.5.1 lib/emily/quantization.ex", quantized_matmul/2 with
// transpose: false, the AWQ layout): y[m][n] = sum_k x[m][k] w_hat[k][n],
// w_hat[k][n] = q[k][n] s[k][g] + b[k][g], g = n / group_size.  For few
// tokens (M <= 16), bits 2, 4 and 8.
//
// Regrouped per column group: within a group the scale and the bias depend
// on k only, so
//   y[m][n] = sum_k (x[m][k] s[k][g]) q[k][n] + sum_k x[m][k] b[k][g],
// one multiply per (k, group) instead of one per code, and the bias term one
// fused multiply-add per (k, group).
//
// Work split.  A cluster of CL CTAs owns 128 consecutive columns; CTA r of
// the cluster walks rows [r Kc, (r + 1) Kc).  In a CTA, 8 threads cover one
// row's 128 columns (16 columns, one group, each) and the 256 threads cover
// 32 rows per step; every thread requests the packed words of kU steps
// before it uses any (enough bytes in flight for HBM: a row's 16 columns
// are only 4 to 16 bytes).  x is staged in shared memory as fp32.  Partial
// sums are reduced over the 32 row slots in a fixed order, then over the
// cluster's ranks in rank order through distributed shared memory by rank 0,
// which stores y: the result does not depend on timing.
#include <algorithm>

#include "common.cuh"

namespace qmm {
namespace t0 {

constexpr int kThreads = 256;
constexpr int kCS = 16;                 // columns per thread (one group: group_size >= 32)
constexpr int kTPR = 8;                 // threads per row
constexpr int kCB = kCS * kTPR;         // columns per cluster
constexpr int kRPI = kThreads / kTPR;   // rows per step
constexpr int kU = 12;                  // steps whose loads are issued together
constexpr int kChunk = 1024;            // rows of x staged at a time

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// all threads of all CTAs of the cluster (a hardware barrier: every thread
// of the cluster reaches it on every path)
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a float of CTA `rank`'s shared memory at the address of `p` in this CTA
__device__ __forceinline__ float ld_peer(const float* p, uint32_t rank) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

// the thread's kCS codes of one row (its packed words) as the floats
// 1024 + code: two codes per 32-bit word at a time under the exponent of an
// f16 pair (one lop3 each, both halves exact), widened to fp32.  The 1024s
// are taken back once per token at the end (1024 times the sum of the x s
// the codes were multiplied by).
template <int B>
__device__ __forceinline__ void codes_1024(const uint32_t* w, float* q) {
  constexpr int CPW = 32 / B;   // codes per word
  constexpr int HALF = CPW / 2; // code j pairs with code j + HALF (the upper 16 bits)
  constexpr uint32_t M = ((1u << B) - 1u) * 0x00010001u;
#pragma unroll
  for (int k = 0; k < kCS / CPW; ++k) {
#pragma unroll
    for (int j = 0; j < HALF; ++j) {
      const uint32_t h = ((w[k] >> (B * j)) & M) | 0x64006400u;
      __half2 hh;
      memcpy(&hh, &h, 4);
      const float2 f = __half22float2(hh);
      q[k * CPW + j] = f.x;
      q[k * CPW + j + HALF] = f.y;
    }
  }
}

template <int B, typename T, int kTok>
__global__ void __launch_bounds__(kThreads)
qgemv_t0_kernel(const T* __restrict__ x, int M, int K, const uint32_t* __restrict__ packed,
                const T* __restrict__ scales, const T* __restrict__ biases, int N, int gs, int kc, void* y,
                int64_t ldy, int y_dtype) {
  constexpr int W = kCS * B / 32;  // packed words of a thread's row segment
  __shared__ float xs[kTok][kChunk];
  __shared__ float red[kTok][kCB][kRPI + 1];  // [token][column][row slot]; slot kRPI: the CTA's sum
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_rank(), ncl = cluster_size();
  const int lw = tid % kTPR, rs = tid / kTPR;
  const int n0 = (int)(blockIdx.x / ncl) * kCB;
  const int ncol = n0 + lw * kCS;
  const bool live = ncol < N;  // N % 16 == 0: a segment is all in or all out
  const int64_t wpr = (int64_t)N * B / 32;
  const int G = N / gs;
  const int g = live ? ncol / gs : 0;
  const int kb = (int)rank * kc, ke = min(K, kb + kc);
  const uint32_t* wbase = packed + (live ? ncol * B / 32 : 0);
  for (int m0 = 0; m0 < M; m0 += kTok) {
    const int mb = min(kTok, M - m0);
    float acc[kTok][kCS], bacc[kTok], sxs[kTok];
#pragma unroll
    for (int t = 0; t < kTok; ++t) {
      bacc[t] = 0.0f;
      sxs[t] = 0.0f;
#pragma unroll
      for (int c = 0; c < kCS; ++c) acc[t][c] = 0.0f;
    }
    for (int k0 = kb; k0 < ke; k0 += kChunk) {
      const int kn = min(kChunk, ke - k0);
      __syncthreads();  // the previous chunk is consumed
      for (int i = tid; i < kTok * kn; i += kThreads) {
        const int t = i / kn, kk = i - t * kn;
        xs[t][kk] = t < mb ? to_f32(x[(int64_t)(m0 + t) * K + k0 + kk]) : 0.0f;
      }
      __syncthreads();
      if (live) {
        for (int kk0 = rs; kk0 < kn; kk0 += kRPI * kU) {
          uint32_t wv[kU][W];
          float sv[kU], bv[kU];
#pragma unroll
          for (int j = 0; j < kU; ++j) {
            const int kk = kk0 + j * kRPI;
            const int64_t k = k0 + (kk < kn ? kk : 0);  // rows past the chunk reread its first row
            const uint32_t* src = wbase + k * wpr;
            if constexpr (W == 4) {
              const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
              wv[j][0] = v.x; wv[j][1] = v.y; wv[j][2] = v.z; wv[j][3] = v.w;
            } else if constexpr (W == 2) {
              const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
              wv[j][0] = v.x; wv[j][1] = v.y;
            } else {
              wv[j][0] = __ldg(src);
            }
            sv[j] = to_f32(scales[k * G + g]);
            bv[j] = to_f32(biases[k * G + g]);
          }
#pragma unroll
          for (int j = 0; j < kU; ++j) {
            const int kk = kk0 + j * kRPI;
            if (kk < kn) {
              float q[kCS];
              codes_1024<B>(wv[j], q);
#pragma unroll
              for (int t = 0; t < kTok; ++t) {
                const float xk = xs[t][kk];
                const float xsk = xk * sv[j];
                bacc[t] = fmaf(xk, bv[j], bacc[t]);
                sxs[t] += xsk;
#pragma unroll
                for (int c = 0; c < kCS; ++c) acc[t][c] = fmaf(xsk, q[c], acc[t][c]);
              }
            }
          }
        }
      }
    }
    // the CTA's sum per (token, column): row slots in increasing order
#pragma unroll
    for (int t = 0; t < kTok; ++t)
#pragma unroll
      for (int c = 0; c < kCS; ++c) red[t][lw * kCS + c][rs] = fmaf(-1024.0f, sxs[t], acc[t][c]) + bacc[t];
    __syncthreads();
    for (int i = tid; i < kTok * kCB; i += kThreads) {
      const int t = i / kCB, c = i - t * kCB;
      float v = 0.0f;
      for (int r = 0; r < kRPI; ++r) v += red[t][c][r];
      red[t][c][kRPI] = v;
    }
    // the cluster's sum: rank 0 adds the ranks' sums in rank order
    cluster_sync();
    if (rank == 0) {
      for (int i = tid; i < kTok * kCB; i += kThreads) {
        const int t = i / kCB, c = i - t * kCB;
        if (t < mb && n0 + c < N) {
          // every rank's sum requested before the first is added
          float pv[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) pv[r] = r < (int)ncl ? ld_peer(&red[t][c][kRPI], (uint32_t)r) : 0.0f;
          float v = 0.0f;
#pragma unroll
          for (int r = 0; r < 8; ++r) v += pv[r];
          store_as(y, y_dtype, (int64_t)(m0 + t) * ldy + n0 + c, v);
        }
      }
    }
    cluster_sync();  // the ranks' sums stay in place until rank 0 has read them
  }
}

template <int B, typename T>
cudaError_t launch_b(const void* x, int64_t M, int64_t K, const qmm_qweight* w, void* y, int64_t ldy, int y_dtype,
                     cudaStream_t st) {
  const int64_t N = w->cols;
  const int sms = qmm_host::num_sms();
  const int nblk = (int)((N + kCB - 1) / kCB);
  // ranks per cluster: split K while the grid stays within two CTAs per SM
  // (one wave at the kernel's register use; at most 8 ranks, at least one
  // step of rows each).  Measured, one token, 4096 x 14336: 2 ranks (224
  // CTAs) -7.5% against 4 ranks (448 CTAs, a second wave).
  int cl = 1;
  while (cl < 8 && (int64_t)nblk * cl * 2 <= 2 * sms && K / (2 * cl) >= kRPI) cl *= 2;
  const int kc = (int)((K + cl - 1) / cl);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nblk * cl));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto k = M == 1 ? qgemv_t0_kernel<B, T, 1> : qgemv_t0_kernel<B, T, 2>;
  return cudaLaunchKernelEx(&cfg, k, reinterpret_cast<const T*>(x), (int)M, (int)K, w->packed,
                            reinterpret_cast<const T*>(w->scales), reinterpret_cast<const T*>(w->biases), (int)N,
                            w->group_size, kc, y, ldy, y_dtype);
}

template <typename T>
cudaError_t launch_t(const void* x, int64_t M, int64_t K, const qmm_qweight* w, void* y, int64_t ldy, int y_dtype,
                     cudaStream_t st) {
  switch (w->bits) {
    case 2: return launch_b<2, T>(x, M, K, w, y, ldy, y_dtype, st);
    case 4: return launch_b<4, T>(x, M, K, w, y, ldy, y_dtype, st);
    default: return launch_b<8, T>(x, M, K, w, y, ldy, y_dtype, st);
  }
}

}  // namespace t0

// cudaErrorNotSupported: not a shape this kernel takes (the caller falls back)
cudaError_t launch_qgemv_t0(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w, void* y,
                            int64_t ldy, int y_dtype, cudaStream_t st) {
  if (M < 1 || M > 16 || (w->bits != 2 && w->bits != 4 && w->bits != 8)) return cudaErrorNotSupported;
  if (K > (int64_t)INT32_MAX || w->cols > (int64_t)INT32_MAX / 8 || w->cols % 16 != 0) return cudaErrorNotSupported;
  // 16-column segments start on a boundary of their load width
  if ((reinterpret_cast<uintptr_t>(w->packed) & 15) != 0) return cudaErrorNotSupported;
  if (x_dtype == QMM_F32) return t0::launch_t<float>(x, M, K, w, y, ldy, y_dtype, st);
  if (x_dtype == QMM_BF16) return t0::launch_t<__nv_bfloat16>(x, M, K, w, y, ldy, y_dtype, st);
  return t0::launch_t<__half>(x, M, K, w, y, ldy, y_dtype, st);
}

}  // namespace qmm
