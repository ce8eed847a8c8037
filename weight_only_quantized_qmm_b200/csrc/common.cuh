// Shared device helpers of the CUDA path (sm_100a).  Nothing here is used by
// the CPU oracle, and nothing here comes from it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "qmm.h"

namespace qmm {

// ---------------------------------------------------------------- dtypes
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// raw 16-bit pattern of a 16-bit float type
__device__ __forceinline__ uint16_t bits16(__nv_bfloat16 v) { return __bfloat16_as_ushort(v); }
__device__ __forceinline__ uint16_t bits16(__half v) { return __half_as_ushort(v); }

// store one fp32 value as out_dtype (runtime choice)
__device__ __forceinline__ void store_as(void* base, int dtype, int64_t idx, float v) {
  if (dtype == QMM_F32)
    reinterpret_cast<float*>(base)[idx] = v;
  else if (dtype == QMM_BF16)
    reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<__half*>(base)[idx] = __float2half_rn(v);
}

// ---------------------------------------------------------------- bit fields
// Code i (compile-time after unrolling) of a register array holding an
// LSB-first bitstream: bits [i*B, i*B+B), possibly spanning two registers.
template <int B>
__device__ __forceinline__ uint32_t stream_code(const uint32_t* r, int i) {
  const int bit = i * B;
  const int w = bit >> 5;
  const int sh = bit & 31;
  uint32_t v;
  if (sh + B <= 32)
    v = r[w] >> sh;
  else
    v = __funnelshift_r(r[w], r[w + 1], sh);
  return v & ((1u << B) - 1u);
}

__device__ __forceinline__ void set_status(int32_t* d_status, int code) {
  if (d_status) atomicOr(d_status, code);
}

}  // namespace qmm

// Host-side helpers shared by the .cu files of the product library.
namespace qmm_host {
inline int dtype_size(qmm_dtype d) { return d == QMM_F32 ? 4 : 2; }
inline bool dtype_ok(int d) { return d == QMM_F32 || d == QMM_F16 || d == QMM_BF16; }
inline bool aligned16(const void* p) { return p && ((reinterpret_cast<uintptr_t>(p) & 15u) == 0); }
int num_sms();
qmm_status launch_status(cudaError_t e);
}  // namespace qmm_host
