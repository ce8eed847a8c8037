// Parameters of the decode-shaped quantized GEMV / MoE kernel family and
// the host helpers that fill them (shared by api.cu and qgemv.cu).
#pragma once

#include "common.cuh"

namespace qmm {

struct QgemvParams {
  const uint32_t* packed[2];
  const void* scales[2];
  const void* biases[2];
  int64_t n_rows;      // rows per expert (N for dense)
  int64_t K;           // reduction length (= quantized cols)
  int64_t wpr;         // packed words per row
  int G;               // groups per row
  int num_experts;     // 1 for dense
  const void* a;
  int amode;           // 0 dense (m*K), 1 p*stride, 2 batched, 3 offset 0
  int64_t stride, outer, inner, top_k;
  const int32_t* ids;  // nullptr for dense
  int n_pairs;
  void* out;
  int out_dtype;
  int64_t out_ld;
  int32_t* d_status;
  int tok_cap;         // tokens per pass (<= 8*MT)
  int kchunk;          // groups staged per K chunk
  int tok_stride;      // bytes between token rows of staged x
  // shared memory carve-up (byte offsets)
  int use_tma;         // 1: take the TMA path when the shape allows it
  int sb_rows;         // rows of the staged scale/bias block
  int sb_words;        // 4-byte words staged per row and array (covers kchunk + 1 elements)
  int off_plan, off_ring, off_part, off_corr, off_xs, off_xsum, off_sb;
};


// Launch planner (qgemv.cu); cudaErrorInvalidValue when a size limit of the
// kernel is exceeded.
cudaError_t launch_qgemv(QgemvParams prm, int bits, int gs, int dtype, bool dual, cudaStream_t st);
// per-tensor dynamic-range int8 [N, K] on the streaming kernel (params from
// make_pt_params); cudaErrorNotSupported when the shape does not fit it
cudaError_t launch_qgemv_pt(const QgemvParams& prm, int dtype, cudaStream_t st);

inline QgemvParams make_dense_params(const void* x, int64_t M, int64_t K, const qmm_qweight* w,
                                     void* y, int64_t ldy, int y_dtype) {
  QgemvParams p{};
  p.packed[0] = w->packed;
  p.scales[0] = w->scales;
  p.biases[0] = w->biases;
  p.n_rows = w->rows;
  p.K = K;
  p.wpr = K * w->bits / 32;
  p.G = (int)(K / w->group_size);
  p.num_experts = 1;
  p.a = x;
  p.amode = 0;
  p.top_k = 1;
  p.ids = nullptr;
  p.n_pairs = (int)M;
  p.out = y;
  p.out_dtype = y_dtype;
  p.out_ld = ldy;
  p.d_status = nullptr;
  p.use_tma = 1;
  return p;
}

// W is int8 [N, K] row-major (as 32-bit words of 4 codes); params: the
// device float[4] {in_min, in_max, out_min, out_max}
inline QgemvParams make_pt_params(const void* x, int64_t M, int64_t K, const int8_t* q, int64_t N,
                                  const float* params, void* y, int y_dtype) {
  QgemvParams p{};
  p.packed[0] = reinterpret_cast<const uint32_t*>(q);
  p.scales[0] = params;
  p.biases[0] = params;
  p.n_rows = N;
  p.K = K;
  p.wpr = K / 4;
  p.G = (int)(K / 64);
  p.num_experts = 1;
  p.a = x;
  p.amode = 0;
  p.top_k = 1;
  p.ids = nullptr;
  p.n_pairs = (int)M;
  p.out = y;
  p.out_dtype = y_dtype;
  p.out_ld = N;
  p.d_status = nullptr;
  p.use_tma = 1;
  return p;
}

inline QgemvParams make_moe_params(const void* a, const int32_t* ids, int64_t n_pairs,
                                   const qmm_expert_stack* w0, const qmm_expert_stack* w1,
                                   void* out, int out_dtype, int32_t* d_status, int amode,
                                   int64_t stride, int64_t outer, int64_t inner, int64_t top_k) {
  QgemvParams p{};
  p.packed[0] = w0->packed;
  p.scales[0] = w0->scales;
  p.biases[0] = w0->biases;
  if (w1) {
    p.packed[1] = w1->packed;
    p.scales[1] = w1->scales;
    p.biases[1] = w1->biases;
  }
  p.n_rows = w0->n_rows;
  p.K = w0->n_cols;
  p.wpr = w0->n_cols * w0->bits / 32;
  p.G = (int)(w0->n_cols / w0->group_size);
  p.num_experts = (int)w0->num_experts;
  p.a = a;
  p.amode = amode;
  p.stride = stride;
  p.outer = outer;
  p.inner = inner;
  p.top_k = top_k;
  p.ids = ids;
  p.n_pairs = (int)n_pairs;
  p.out = out;
  p.out_dtype = out_dtype;
  p.out_ld = w0->n_rows;
  p.d_status = d_status;
  p.use_tma = 1;
  return p;
}

}  // namespace qmm
