// C ABI of libqmm.so: argument validation and kernel dispatch.  Every entry
// point validates on the host, returns a qmm_status, launches asynchronously
// on the caller's stream and never synchronizes or allocates.
#include <stdio.h>

#include <algorithm>

#include "common.cuh"

namespace qmm {
cudaError_t launch_quantize(int w_dtype, int s_dtype, int bits, const void* w, int64_t rows,
                            int64_t cols, int gs, uint32_t* packed, void* scales, void* biases,
                            cudaStream_t st);
cudaError_t launch_dequantize(const qmm_qweight* w, void* out, int out_dtype, cudaStream_t st);
cudaError_t launch_generic(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w,
                           int transpose, void* y, int64_t ldy, int y_dtype, cudaStream_t st);
cudaError_t launch_qgemm_tc(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w,
                            void* y, int64_t ldy, int y_dtype, cudaStream_t st);
cudaError_t launch_dequantize_mx(const qmm_qweight* w, void* out, int out_dtype, cudaStream_t st);
cudaError_t launch_matmul_mx(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w, void* y,
                             int64_t ldy, int y_dtype, cudaStream_t st);
cudaError_t launch_qgemv_t0(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w, void* y,
                            int64_t ldy, int y_dtype, cudaStream_t st);
cudaError_t launch_quantize_dyn8(const void* w, int w_dtype, int64_t n, int8_t* q, float* params, cudaStream_t st);
cudaError_t launch_dequantize_dyn8(const int8_t* q, int64_t n, const float* params, void* out, int out_dtype,
                                   cudaStream_t st);
cudaError_t launch_matmul_dyn8(const void* x, int x_dtype, int64_t M, int64_t K, const int8_t* q, int64_t N,
                               const float* params, void* y, int y_dtype, cudaStream_t st);
}  // namespace qmm

#include "qgemv.cuh"

namespace qmm_host {

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

qmm_status launch_status(cudaError_t e) { return e == cudaSuccess ? QMM_OK : QMM_ERR_CUDA; }

static bool bits_ok(int b) { return b == 2 || b == 3 || b == 4 || b == 6 || b == 8; }
static bool gs_ok(int g) { return g == 32 || g == 64 || g == 128; }
static bool packable(int64_t cols, int gs, int bits) {
  return bits_ok(bits) && gs_ok(gs) && cols > 0 && cols % gs == 0 && (cols * bits) % 32 == 0;
}
static bool aligned4(const void* p) { return p && ((reinterpret_cast<uintptr_t>(p) & 3u) == 0); }

// Largest MoE call the kernels' per-CTA plans are sized for (pairs, experts).
constexpr int64_t kMaxMoePairs = 65536;
// Most parts of one fused projection.
constexpr int kMaxParts = 64;

// m * top_k pairs of a batched MoE call; a product above kMaxMoePairs is
// reported as kMaxMoePairs + 1 (rejected as unsupported) without overflowing.
static int64_t batched_pairs(int64_t m, int64_t top_k) {
  return (m > 0 && top_k > kMaxMoePairs / m) ? kMaxMoePairs + 1 : m * top_k;
}

// bits and group size of a microscaled mode (false for any other mode)
static bool mx_params(int mode, int* bits, int* gs) {
  switch (mode) {
    case QMM_MODE_MXFP4: *bits = 4; *gs = 32; return true;
    case QMM_MODE_MXFP8: *bits = 8; *gs = 32; return true;
    case QMM_MODE_NVFP4: *bits = 4; *gs = 16; return true;
    default: return false;
  }
}

static qmm_status check_qweight(const qmm_qweight* w) {
  if (!w) return QMM_ERR_INVALID_ARG;
  if (w->mode != QMM_MODE_AFFINE) {
    int bits = 0, gs = 0;
    if (!mx_params(w->mode, &bits, &gs)) return QMM_ERR_UNSUPPORTED;
    if (w->sdtype != QMM_U8) return QMM_ERR_DTYPE;
    if (w->bits != bits || w->group_size != gs || w->rows < 0 || w->cols <= 0 || w->cols % 32 != 0)
      return QMM_ERR_INVALID_ARG;
    if (!aligned16(w->packed) || !aligned16(w->scales)) return QMM_ERR_ALIGNMENT;
    return QMM_OK;
  }
  if (!dtype_ok(w->sdtype)) return QMM_ERR_DTYPE;
  if (w->rows < 0 || !packable(w->cols, w->group_size, w->bits)) return QMM_ERR_INVALID_ARG;
  if (!aligned16(w->packed) || !aligned16(w->scales) || !aligned16(w->biases)) return QMM_ERR_ALIGNMENT;
  return QMM_OK;
}

static qmm_status check_stack(const qmm_expert_stack* w) {
  if (!w) return QMM_ERR_INVALID_ARG;
  if (!dtype_ok(w->sdtype)) return QMM_ERR_DTYPE;
  if (w->num_experts < 1 || w->n_rows < 1 || !packable(w->n_cols, w->group_size, w->bits))
    return QMM_ERR_INVALID_ARG;
  if (!aligned16(w->packed) || !aligned16(w->scales) || !aligned16(w->biases)) return QMM_ERR_ALIGNMENT;
  return QMM_OK;
}

static qmm_status device_check() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QMM_ERR_CUDA;
  static int cached[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev] == 1 ? QMM_OK : QMM_ERR_UNSUPPORTED;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return QMM_ERR_CUDA;
  const bool ok = (major == 10 && minor == 0);
  if (dev >= 0 && dev < 64) cached[dev] = ok ? 1 : 2;
  return ok ? QMM_OK : QMM_ERR_UNSUPPORTED;
}

}  // namespace qmm_host

using namespace qmm_host;

extern "C" {

int64_t qmm_packed_words_per_row(int64_t cols, int bits) {
  if (!bits_ok(bits) || cols <= 0 || (cols * bits) % 32 != 0) return -1;
  return cols * bits / 32;
}

int64_t qmm_groups_per_row(int64_t cols, int group_size) {
  if (!gs_ok(group_size) || cols <= 0 || cols % group_size != 0) return -1;
  return cols / group_size;
}

const char* qmm_status_string(int s) {
  switch (s) {
    case QMM_OK: return "ok";
    case QMM_ERR_INVALID_ARG: return "invalid argument (bits, group_size, shape, mode or flag)";
    case QMM_ERR_UNSUPPORTED: return "unsupported (mode, device or size limit)";
    case QMM_ERR_DTYPE: return "dtype rule violated (input dtype must match scales dtype)";
    case QMM_ERR_ALIGNMENT: return "null or under-aligned pointer";
    case QMM_ERR_CUDA: return "CUDA runtime error";
    case QMM_ERR_TIMEOUT: return "device-side wait timed out";
    case QMM_ERR_BAD_EXPERT_ID: return "expert id out of range";
    default: return "unknown status";
  }
}

qmm_status qmm_device_check(void) { return device_check(); }

qmm_status qmm_quantize(const void* w, qmm_dtype w_dtype, int64_t rows, int64_t cols,
                        int group_size, int bits, qmm_dtype s_dtype, uint32_t* packed,
                        void* scales, void* biases, void* stream) {
  if (!dtype_ok(w_dtype) || !dtype_ok(s_dtype)) return QMM_ERR_DTYPE;
  if (rows < 0 || !packable(cols, group_size, bits)) return QMM_ERR_INVALID_ARG;
  if (rows == 0) return QMM_OK;
  if (!aligned16(w) || !aligned16(packed) || !aligned16(scales) || !aligned16(biases))
    return QMM_ERR_ALIGNMENT;
  qmm_status s = device_check();
  if (s != QMM_OK) return s;
  return launch_status(qmm::launch_quantize(w_dtype, s_dtype, bits, w, rows, cols, group_size,
                                            packed, scales, biases, (cudaStream_t)stream));
}

qmm_status qmm_dequantize(const qmm_qweight* w, void* out, qmm_dtype out_dtype, void* stream) {
  qmm_status s = check_qweight(w);
  if (s != QMM_OK) return s;
  if (!dtype_ok(out_dtype)) return QMM_ERR_DTYPE;
  if (w->rows == 0) return QMM_OK;
  if (!aligned16(out)) return QMM_ERR_ALIGNMENT;
  s = device_check();
  if (s != QMM_OK) return s;
  if (w->mode != QMM_MODE_AFFINE)
    return launch_status(qmm::launch_dequantize_mx(w, out, out_dtype, (cudaStream_t)stream));
  return launch_status(qmm::launch_dequantize(w, out, out_dtype, (cudaStream_t)stream));
}

// argument rules of qmm_matmul for one weight (no launch)
static qmm_status check_matmul(qmm_dtype x_dtype, int64_t M, int64_t K, const qmm_qweight* w, int transpose,
                               qmm_dtype y_dtype) {
  qmm_status s = check_qweight(w);
  if (s != QMM_OK) return s;
  if (transpose != 0 && transpose != 1) return QMM_ERR_INVALID_ARG;
  if (!dtype_ok(x_dtype) || !dtype_ok(y_dtype)) return QMM_ERR_DTYPE;
  // affine: x and the scales share a dtype; microscaled: any float x
  if (w->mode == QMM_MODE_AFFINE && x_dtype != w->sdtype) return QMM_ERR_DTYPE;
  if (y_dtype != x_dtype && y_dtype != QMM_F32) return QMM_ERR_DTYPE;
  if (w->mode != QMM_MODE_AFFINE && !transpose) return QMM_ERR_UNSUPPORTED;
  if (M < 0 || K <= 0) return QMM_ERR_INVALID_ARG;
  if ((transpose ? w->cols : w->rows) != K) return QMM_ERR_INVALID_ARG;
  return QMM_OK;
}

// the kernel choice of qmm_matmul; y rows are ldy elements apart
static qmm_status matmul_dispatch(const void* x, qmm_dtype x_dtype, int64_t M, int64_t K, const qmm_qweight* w,
                                  int transpose, void* y, int64_t ldy, qmm_dtype y_dtype, cudaStream_t st) {
  if (w->mode != QMM_MODE_AFFINE)
    return launch_status(qmm::launch_matmul_mx(x, x_dtype, M, K, w, y, ldy, y_dtype, st));
  const bool half_types = (x_dtype == QMM_BF16 || x_dtype == QMM_F16);
  if (transpose && half_types && M <= 16) {
    qmm::QgemvParams p = qmm::make_dense_params(x, M, K, w, y, ldy, y_dtype);
    const cudaError_t e = qmm::launch_qgemv(p, w->bits, w->group_size, x_dtype, false, st);
    if (e == cudaErrorInvalidValue) return QMM_ERR_UNSUPPORTED;
    return launch_status(e);
  }
  if (transpose && half_types) {  // M > 16: tcgen05 tensor-core GEMM
    const cudaError_t e = qmm::launch_qgemm_tc(x, x_dtype, M, K, w, y, ldy, y_dtype, st);
    if (e != cudaErrorNotSupported) return launch_status(e);
  }
  if (!transpose) {  // [K, N] weights, few tokens, whole-word codes
    const cudaError_t e = qmm::launch_qgemv_t0(x, x_dtype, M, K, w, y, ldy, y_dtype, st);
    if (e != cudaErrorNotSupported) return launch_status(e);
  }
  return launch_status(qmm::launch_generic(x, x_dtype, M, K, w, transpose, y, ldy, y_dtype, st));
}

qmm_status qmm_matmul(const void* x, qmm_dtype x_dtype, int64_t M, int64_t K,
                      const qmm_qweight* w, int transpose, void* y, qmm_dtype y_dtype,
                      void* stream) {
  qmm_status s = check_matmul(x_dtype, M, K, w, transpose, y_dtype);
  if (s != QMM_OK) return s;
  const int64_t N = transpose ? w->rows : w->cols;
  if (M == 0 || N == 0) return QMM_OK;
  if (!aligned16(x) || !aligned16(y)) return QMM_ERR_ALIGNMENT;
  s = device_check();
  if (s != QMM_OK) return s;
  return matmul_dispatch(x, x_dtype, M, K, w, transpose, y, N, y_dtype, (cudaStream_t)stream);
}

qmm_status qmm_matmul_parts(const void* x, qmm_dtype x_dtype, int64_t M, int64_t K, const qmm_qweight* parts,
                            int n_parts, void* y, qmm_dtype y_dtype, void* stream) {
  if (!parts || n_parts < 1 || n_parts > kMaxParts) return QMM_ERR_INVALID_ARG;
  int64_t ldy = 0;
  for (int i = 0; i < n_parts; ++i) {
    const qmm_status s = check_matmul(x_dtype, M, K, &parts[i], 1, y_dtype);
    if (s != QMM_OK) return s;
    ldy += parts[i].rows;
  }
  if (M == 0 || ldy == 0) return QMM_OK;
  if (!aligned16(x) || !aligned16(y)) return QMM_ERR_ALIGNMENT;
  qmm_status s = device_check();
  if (s != QMM_OK) return s;
  const int esize = y_dtype == QMM_F32 ? 4 : 2;
  int64_t off = 0;
  for (int i = 0; i < n_parts; ++i) {
    if (parts[i].rows > 0) {
      s = matmul_dispatch(x, x_dtype, M, K, &parts[i], 1, static_cast<char*>(y) + off * esize, ldy, y_dtype,
                          (cudaStream_t)stream);
      if (s != QMM_OK) return s;
    }
    off += parts[i].rows;
  }
  return QMM_OK;
}

qmm_status qmm_quantize_dynamic_int8(const void* w, qmm_dtype w_dtype, int64_t n, int8_t* q, float* params,
                                     void* stream) {
  if (!dtype_ok(w_dtype)) return QMM_ERR_DTYPE;
  if (n <= 0) return QMM_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(q) || !aligned4(params)) return QMM_ERR_ALIGNMENT;
  const qmm_status s = device_check();
  if (s != QMM_OK) return s;
  return launch_status(qmm::launch_quantize_dyn8(w, w_dtype, n, q, params, (cudaStream_t)stream));
}

qmm_status qmm_dequantize_dynamic_int8(const int8_t* q, int64_t n, const float* params, void* out,
                                       qmm_dtype out_dtype, void* stream) {
  if (!dtype_ok(out_dtype)) return QMM_ERR_DTYPE;
  if (n < 0) return QMM_ERR_INVALID_ARG;
  if (n == 0) return QMM_OK;
  if (!aligned16(q) || !aligned16(out) || !aligned4(params)) return QMM_ERR_ALIGNMENT;
  const qmm_status s = device_check();
  if (s != QMM_OK) return s;
  return launch_status(qmm::launch_dequantize_dyn8(q, n, params, out, out_dtype, (cudaStream_t)stream));
}

qmm_status qmm_matmul_dynamic_int8(const void* x, qmm_dtype x_dtype, int64_t M, int64_t K, const int8_t* q,
                                   int64_t N, const float* params, void* y, qmm_dtype y_dtype, void* stream) {
  if (!dtype_ok(x_dtype) || !dtype_ok(y_dtype)) return QMM_ERR_DTYPE;
  if (y_dtype != x_dtype && y_dtype != QMM_F32) return QMM_ERR_DTYPE;
  if (M < 0 || K <= 0 || N < 0) return QMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return QMM_OK;
  if (!aligned16(x) || !aligned16(q) || !aligned16(y) || !aligned4(params)) return QMM_ERR_ALIGNMENT;
  const qmm_status s = device_check();
  if (s != QMM_OK) return s;
  // few tokens, 16-bit x, rows of whole 32-group units (K % 512 == 0,
  // K >= 2048): the streaming tensor-core GEMV with the per-tensor scale
  if ((x_dtype == QMM_BF16 || x_dtype == QMM_F16) && M <= 16 && K % 512 == 0 && K >= 2048 &&
      K <= (int64_t)INT32_MAX && N >= 16) {
    const qmm::QgemvParams p = qmm::make_pt_params(x, M, K, q, N, params, y, y_dtype);
    const cudaError_t e = qmm::launch_qgemv_pt(p, x_dtype, (cudaStream_t)stream);
    if (e != cudaErrorNotSupported) return launch_status(e);
  }
  return launch_status(qmm::launch_matmul_dyn8(x, x_dtype, M, K, q, N, params, y, y_dtype, (cudaStream_t)stream));
}

static qmm_status moe_common(const void* a, qmm_dtype a_dtype, const int32_t* ids,
                             int64_t n_pairs, const qmm_expert_stack* w0,
                             const qmm_expert_stack* w1, void* out, qmm_dtype out_dtype,
                             int32_t* d_status, void* stream, int amode, int64_t stride,
                             int64_t outer, int64_t inner, int64_t top_k) {
  qmm_status s = check_stack(w0);
  if (s != QMM_OK) return s;
  if (w1) {
    s = check_stack(w1);
    if (s != QMM_OK) return s;
    if (w1->num_experts != w0->num_experts || w1->n_rows != w0->n_rows ||
        w1->n_cols != w0->n_cols || w1->group_size != w0->group_size || w1->bits != w0->bits ||
        w1->sdtype != w0->sdtype)
      return QMM_ERR_INVALID_ARG;
  }
  if (!dtype_ok(a_dtype) || !dtype_ok(out_dtype)) return QMM_ERR_DTYPE;
  if (a_dtype != w0->sdtype) return QMM_ERR_DTYPE;
  if (out_dtype != a_dtype && out_dtype != QMM_F32) return QMM_ERR_DTYPE;
  if (n_pairs < 0 || stride < 0 || outer < 0 || inner < 0) return QMM_ERR_INVALID_ARG;
  if (n_pairs == 0) return QMM_OK;
  if (a_dtype == QMM_F32) return QMM_ERR_UNSUPPORTED;  // tensor-core path only
  if (n_pairs > kMaxMoePairs || w0->num_experts > kMaxMoePairs) return QMM_ERR_UNSUPPORTED;
  if (!a || (reinterpret_cast<uintptr_t>(a) & 1u)) return QMM_ERR_ALIGNMENT;
  if (!aligned4(ids) || !aligned16(out)) return QMM_ERR_ALIGNMENT;
  if (d_status && !aligned4(d_status)) return QMM_ERR_ALIGNMENT;
  s = device_check();
  if (s != QMM_OK) return s;
  qmm::QgemvParams p = qmm::make_moe_params(a, ids, n_pairs, w0, w1, out, out_dtype, d_status,
                                            amode, stride, outer, inner, top_k);
  const cudaError_t e =
      qmm::launch_qgemv(p, w0->bits, w0->group_size, a_dtype, w1 != nullptr, (cudaStream_t)stream);
  if (e == cudaErrorInvalidValue) return QMM_ERR_UNSUPPORTED;
  return launch_status(e);
}

qmm_status qmm_moe_gemv_id(const void* a, qmm_dtype a_dtype, const int32_t* ids,
                           int64_t n_selected, int64_t src1_stride, const qmm_expert_stack* w,
                           void* out, qmm_dtype out_dtype, int32_t* d_status, void* stream) {
  return moe_common(a, a_dtype, ids, n_selected, w, nullptr, out, out_dtype, d_status, stream, 1,
                    src1_stride, 0, 0, 1);
}

qmm_status qmm_moe_gemv_id_batched(const void* a, qmm_dtype a_dtype, const int32_t* ids,
                                   int64_t m, int64_t top_k, int64_t outer_stride,
                                   int64_t inner_stride, const qmm_expert_stack* w, void* out,
                                   qmm_dtype out_dtype, int32_t* d_status, void* stream) {
  if (m < 0 || top_k <= 0) return QMM_ERR_INVALID_ARG;
  return moe_common(a, a_dtype, ids, batched_pairs(m, top_k), w, nullptr, out, out_dtype, d_status, stream, 2,
                    0, outer_stride, inner_stride, top_k);
}

qmm_status qmm_moe_gemv_id_gate_up_silu(const void* a, qmm_dtype a_dtype, const int32_t* ids,
                                        int64_t n_selected, const qmm_expert_stack* gate,
                                        const qmm_expert_stack* up, void* silu_out,
                                        qmm_dtype out_dtype, int32_t* d_status, void* stream) {
  if (!up) return QMM_ERR_INVALID_ARG;
  return moe_common(a, a_dtype, ids, n_selected, gate, up, silu_out, out_dtype, d_status, stream,
                    3, 0, 0, 0, 1);
}

qmm_status qmm_moe_gemv_id_gate_up_silu_batched(const void* a, qmm_dtype a_dtype,
                                                const int32_t* ids, int64_t m, int64_t top_k,
                                                int64_t outer_stride, int64_t inner_stride,
                                                const qmm_expert_stack* gate,
                                                const qmm_expert_stack* up, void* silu_out,
                                                qmm_dtype out_dtype, int32_t* d_status,
                                                void* stream) {
  if (!up) return QMM_ERR_INVALID_ARG;
  if (m < 0 || top_k <= 0) return QMM_ERR_INVALID_ARG;
  return moe_common(a, a_dtype, ids, batched_pairs(m, top_k), gate, up, silu_out, out_dtype, d_status, stream,
                    2, 0, outer_stride, inner_stride, top_k);
}

}  // extern "C"
