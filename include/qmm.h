/*
 * qmm.h -- C ABI of libqmm.so: weight-only quantized matmul on NVIDIA B200
 * (sm_100a): affine, microscaled and per-tensor int8 weights.
 *
 * What is computed (sources cited by page title and section):
 *   - Packed weights: b-bit codes (b in {2,3,4,6,8}) stored LSB-first along
 *     the row in little-endian uint32 words; code i of a row sits at stream
 *     bits [i*b, (i+1)*b) and may straddle two words when b is 3 or 6
 *     ("emily 0.5.1 lib/emily/quantization.ex", dequantize_defn/1,
 *     unpack_integral_lanes, unpack_cross_word_lanes).
 *   - Affine dequantization: w_hat[r][i] = q * scale[r][g] + bias[r][g],
 *     g = i / group_size (same page, dequantize_defn/1 doc).  This library
 *     evaluates it as one fp32 fused multiply-add.
 *   - Quantized matmul: y = x . dequant(W)^T for transpose = 1, the AWQ
 *     layout y = x . dequant(W) for transpose = 0 (same page,
 *     quantized_matmul/2); affine mode requires x and the scales to share a
 *     dtype (same page, validate_dtype_match!).
 *   - MoE stacked experts: out[i] = a[off(i)] . dequant(W[ids[i]])^T and the
 *     fused SiLU(gate) * up form, single and batched
 *     ("ferrum-kernels 0.7.7 src/stacked_expert.rs", StackedExpertGgufLinear:
 *     gemv_moe_id, gemv_moe_id_batched, gemv_moe_id_gate_up_silu,
 *     gemv_moe_id_gate_up_silu_batched).  The offset-aware form
 *     (gemv_moe_id_offset) is the same call with `a` and `ids` advanced by
 *     the caller.
 *   - Quantizer: per (row, group) min/max; the page that calls it
 *     ("ollama x/create/client/quantize.go", loadAndQuantizeArray) does not
 *     print its body, so this library uses the min/max rule of
 *     "mlex 0.1.3 src/quant.rs" quantize_dynamic_int8 applied per group:
 *     scale = max((max-min)/(2^b-1), FLT_EPSILON), bias = min,
 *     q = clamp(round_half_away((w - bias)/scale), 0, 2^b-1), with scale and
 *     bias first rounded to the scales dtype.
 *
 * Conventions for every call:
 *   - All buffer pointers are DEVICE pointers owned by the caller; the
 *     library keeps no allocation across calls and allocates nothing.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronizes the host.
 *   - Host-side argument errors are returned before anything is launched.
 *     Errors found on the device (a bad expert id; QMM_ERR_TIMEOUT when a
 *     bounded wait inside a kernel gave up) are OR-ed into *d_status (a
 *     caller-zeroed device int32, may be NULL), read by the caller after the
 *     stream has synchronized.  qmm_matmul takes no status buffer: there a
 *     device-side timeout leaves y incomplete (the prefill GEMM writes the
 *     affected tile as NaN).  The library never aborts and never waits
 *     without a bound.
 *   - Shapes: group_size in {32, 64, 128}; cols % group_size == 0 and
 *     cols * bits % 32 == 0 for the quantized axis.
 *   - Alignment: packed, scales, biases, x, y and out must be 16-byte
 *     aligned (QMM_ERR_ALIGNMENT otherwise); MoE activation rows `a + off`
 *     only need element alignment.
 *   - Requires a compute-capability 10.0 device (QMM_ERR_UNSUPPORTED
 *     otherwise).
 *   - MoE calls: a_dtype must be QMM_BF16 or QMM_F16 (QMM_F32 activations
 *     are QMM_ERR_UNSUPPORTED); ids and d_status must be 4-byte aligned; a
 *     negative stride, pair count or m, or top_k <= 0, is
 *     QMM_ERR_INVALID_ARG.  These are decode-size kernels: every CTA keeps
 *     the call's expert plan (two ints per pair, four or five per expert) in
 *     shared memory beside its pipeline buffers, so the pair count
 *     (n_selected, or m * top_k) that fits depends on num_experts and the
 *     kernel.  At 128 experts that is about 3,800 pairs for the fused
 *     gate/up calls and about 6,800 for the single ones.  A larger call, or
 *     one with more than 65536 pairs or experts, returns
 *     QMM_ERR_UNSUPPORTED before anything is launched.
 */
#ifndef QMM_H_
#define QMM_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QMM_OK = 0,
  QMM_ERR_INVALID_ARG = 1,   /* bad bits/group_size/shape/mode/flag */
  QMM_ERR_UNSUPPORTED = 2,   /* non-affine mode, unsupported device or size */
  QMM_ERR_DTYPE = 3,         /* dtype rule violated (x vs scales, out dtype) */
  QMM_ERR_ALIGNMENT = 4,     /* null or under-aligned pointer */
  QMM_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
  QMM_ERR_TIMEOUT = 6,       /* a bounded device-side wait gave up */
  QMM_ERR_BAD_EXPERT_ID = 7  /* (device) an id outside [0, num_experts) */
} qmm_status;

/* QMM_U8 is only the storage of the microscaled modes' scale bytes. */
typedef enum { QMM_F32 = 0, QMM_F16 = 1, QMM_BF16 = 2, QMM_U8 = 3 } qmm_dtype;

/* Quantization modes ("emily 0.5.1 lib/emily/quantization.ex", the modes of
 * dequantize_defn/1, with the group sizes of "ollama
 * x/create/client/quantize.go" quantizeParams):
 *   AFFINE: b-bit codes, w = q * scale + bias per group (scales/biases in the
 *           activation dtype);
 *   MXFP4:  bits 4, group 32: FP4-E2M1 lanes times an FP8-E8M0 scale byte
 *           (2^(s - 127));
 *   MXFP8:  bits 8, group 32: FP8-E4M3 lanes times an E8M0 scale byte;
 *   NVFP4:  bits 4, group 16: FP4-E2M1 lanes times an FP8-E4M3 scale byte.
 * The E4M3 decode is the page's: the low 7 bits shifted left by 7 read as a
 * binary16, times 256, sign from bit 7 (0x7F and 0xFF read as +-480, not
 * NaN).  A microscaled qmm_qweight has sdtype QMM_U8, scales [rows,
 * cols/group_size] uint8, biases unused (may be NULL), and bits/group_size
 * equal to the mode's (QMM_ERR_INVALID_ARG otherwise); w_hat = lane * scale
 * in fp32.  The microscaled modes are served by qmm_dequantize and
 * qmm_matmul (transpose = 1, any float x); qmm_quantize and the MoE calls
 * are affine only (the pages print no quantizer for these modes). */
typedef enum {
  QMM_MODE_AFFINE = 0,
  QMM_MODE_MXFP4 = 1,
  QMM_MODE_MXFP8 = 2,
  QMM_MODE_NVFP4 = 3
} qmm_mode;

/* A quantized matrix ("emily" %QuantizedWeight{value, scales, biases,
 * group_size, bits, mode}).  packed: [rows, cols*bits/32] uint32 row-major;
 * scales, biases: [rows, cols/group_size] row-major in `sdtype`.  The
 * quantized axis is `cols`. */
typedef struct {
  const uint32_t* packed;
  const void* scales;
  const void* biases;
  qmm_dtype sdtype;
  int64_t rows;
  int64_t cols;
  int group_size;
  int bits;
  qmm_mode mode;
} qmm_qweight;

/* N experts of one role (gate, up or down) stored contiguously ("ferrum"
 * StackedExpertGgufLinear): expert e is rows [e*n_rows, (e+1)*n_rows) of
 * packed [num_experts*n_rows, n_cols*bits/32] and of scales/biases
 * [num_experts*n_rows, n_cols/group_size]. */
typedef struct {
  const uint32_t* packed;
  const void* scales;
  const void* biases;
  qmm_dtype sdtype;
  int64_t num_experts;
  int64_t n_rows;
  int64_t n_cols;
  int group_size;
  int bits;
} qmm_expert_stack;

/* cols*bits/32, or -1 when (cols, bits) cannot be packed without a partial
 * word (bits not in {2,3,4,6,8}, cols <= 0, or cols*bits % 32 != 0). */
int64_t qmm_packed_words_per_row(int64_t cols, int bits);

/* cols/group_size, or -1 (group_size not in {32,64,128}, cols % gs != 0). */
int64_t qmm_groups_per_row(int64_t cols, int group_size);

/* Static English text for a status code (never NULL). */
const char* qmm_status_string(int status);

/* QMM_OK when the current CUDA device is compute capability 10.0. */
qmm_status qmm_device_check(void);

/* Dense -> (packed, scales, biases): the quantize step that "ollama
 * x/create/client/quantize.go" (loadAndQuantizeArray) calls, with the
 * per-group min/max rule of the quantizer paragraph above.
 * w: [rows, cols] row-major in w_dtype (f32, f16 or bf16).  packed:
 * [rows, cols*bits/32] uint32; scales, biases: [rows, cols/group_size] in
 * s_dtype.  Bit-exact, whatever the launch shape.  rows == 0 is a no-op.
 * Errors: INVALID_ARG for bits, group_size or cols outside the shape rules
 * or rows < 0; DTYPE for an unknown dtype; ALIGNMENT for a null or
 * under-aligned pointer; UNSUPPORTED on a device that is not compute
 * capability 10.0; CUDA when the launch fails. */
qmm_status qmm_quantize(const void* w, qmm_dtype w_dtype, int64_t rows, int64_t cols,
                        int group_size, int bits, qmm_dtype s_dtype, uint32_t* packed,
                        void* scales, void* biases, void* stream);

/* Standalone dequantization ("emily 0.5.1 lib/emily/quantization.ex",
 * dequantize_defn/1): out[r][i] = fmaf(q, scale, bias) (affine) or
 * lane(q) * scale (microscaled), stored in out_dtype with one RNE rounding
 * for f16/bf16 and none for f32.  out: [w->rows, w->cols] row-major.
 * Bit-exact.  w->rows == 0 is a no-op.
 * Errors: INVALID_ARG (shape rules, null w), UNSUPPORTED (an unknown mode,
 * or the device), DTYPE, ALIGNMENT, CUDA. */
qmm_status qmm_dequantize(const qmm_qweight* w, void* out, qmm_dtype out_dtype, void* stream);

/* Quantized matmul ("emily 0.5.1 lib/emily/quantization.ex",
 * quantized_matmul/2):
 * y[M, N] = x[M, K] . dequant(W)^T  (transpose = 1: W is [N, K], w->rows = N,
 *                                    w->cols = K)
 * y[M, N] = x[M, K] . dequant(W)    (transpose = 0: W is [K, N] quantized
 *                                    along N, w->rows = K, w->cols = N)
 * x_dtype must equal w->sdtype; y_dtype is x_dtype or QMM_F32 (same
 * arithmetic, different final store).  x: [M, K] row-major; y: [M, N]
 * row-major.  Accumulation is fp32.  M == 0 is a no-op.  bf16/f16 with
 * transpose = 1 use the tensor-core kernels (M <= 16: the streaming GEMV;
 * M > 16: the tcgen05 GEMM).
 * Microscaled modes take any float x, transpose = 1 only.
 * Errors: INVALID_ARG (shape rules, K != the weight's input dimension,
 * transpose not 0/1, M < 0), UNSUPPORTED (an unknown mode, a microscaled
 * mode with transpose = 0, or a device that is not compute capability
 * 10.0), DTYPE (affine x_dtype != w->sdtype, or y_dtype neither x_dtype nor
 * f32), ALIGNMENT, CUDA. */
qmm_status qmm_matmul(const void* x, qmm_dtype x_dtype, int64_t M, int64_t K,
                      const qmm_qweight* w, int transpose, void* y, qmm_dtype y_dtype,
                      void* stream);

/* Fused projection over parts that share the input dimension
 * ("ferrum-quantization 0.7.2 src/quant_linear.rs", QuantLinear::
 * from_gguf_fused: each part keeps its own storage and quantization
 * parameters, and the forward pass is one matvec per part):
 * y[:, off_p : off_p + N_p] = x . dequant(W_p)^T for p in [0, n_parts),
 * N_p = parts[p].rows, off_p = N_0 + ... + N_{p-1}; y is [M, sum N_p]
 * row-major.  Parts may differ in bits, group size and mode; each one
 * follows qmm_matmul's rules with transpose = 1 and runs the kernel
 * qmm_matmul picks for it, writing its columns of y in place (no
 * concatenated copy of the weights or of the outputs).
 * Errors: INVALID_ARG (parts NULL, n_parts outside [1, 64], or any part
 * breaking qmm_matmul's rules), the other qmm_matmul errors per part.  All
 * parts are checked before the first launch; a launch failure returns at
 * once with the earlier parts already queued on the stream. */
qmm_status qmm_matmul_parts(const void* x, qmm_dtype x_dtype, int64_t M, int64_t K,
                            const qmm_qweight* parts, int n_parts, void* y, qmm_dtype y_dtype,
                            void* stream);

/* Per-tensor dynamic-range int8 ("mlex 0.1.3 src/quant.rs",
 * DynamicRangeParams, quantize_dynamic_int8, dequantize_dynamic_int8): one
 * scale and zero point for a whole tensor.  params is a DEVICE float[4]
 * {input_min, input_max, output_min, output_max} (4-byte aligned); the
 * codes q are int8 in the tensor's own layout (a [N, K] weight is N*K codes,
 * row-major).
 *   w_hat = fl(fl(fl(q + 128) * scale) + output_min),
 *   scale = fl((output_max - output_min) / 255)     (fp32, three roundings)
 *
 * qmm_quantize_dynamic_int8: params = {min, max, min, max} of the n elements
 * of w (a fold from +-infinity that passes over NaN), then
 * q = clamp(round_half_away((w - min) / s) - 128, -128, 127) with
 * s = max((max - min) / 255, FLT_EPSILON), every step in fp32; a NaN
 * element gets code 0.  Bit-exact.  Four kernels on `stream` (min/max
 * reduction through params, codes, params).
 * Errors: DTYPE (w_dtype), INVALID_ARG (n <= 0), ALIGNMENT (w, q 16-byte;
 * params 4-byte), UNSUPPORTED (device), CUDA. */
qmm_status qmm_quantize_dynamic_int8(const void* w, qmm_dtype w_dtype, int64_t n, int8_t* q,
                                     float* params, void* stream);

/* out[i] = w_hat(q[i]) stored in out_dtype (one RNE rounding for f16/bf16).
 * Bit-exact.  n == 0 is a no-op.
 * Errors: DTYPE, INVALID_ARG (n < 0), ALIGNMENT (q, out 16-byte; params
 * 4-byte), UNSUPPORTED, CUDA. */
qmm_status qmm_dequantize_dynamic_int8(const int8_t* q, int64_t n, const float* params, void* out,
                                       qmm_dtype out_dtype, void* stream);

/* y[M, N] = x[M, K] . w_hat^T for an int8 weight q [N, K] (row-major), any
 * float x; y_dtype is x_dtype or QMM_F32.  fp32 accumulation, the row dot
 * regrouped as scale * sum x (q + 128) + output_min * sum x (M <= 16 with
 * 16-bit x, K a multiple of 512 and N >= 16: the tensor-core streaming
 * kernel: q + 128 exact in f16, x rounded to f16 after a power-of-two
 * scaling per 64 values that puts their largest magnitude in [2^14, 2^15)).
 * M == 0 or N == 0 is a no-op.
 * Errors: DTYPE, INVALID_ARG (M < 0, K <= 0, N < 0), ALIGNMENT (x, q, y
 * 16-byte; params 4-byte), UNSUPPORTED, CUDA. */
qmm_status qmm_matmul_dynamic_int8(const void* x, qmm_dtype x_dtype, int64_t M, int64_t K,
                                   const int8_t* q, int64_t N, const float* params, void* y,
                                   qmm_dtype y_dtype, void* stream);

/* MoE indirect GEMV ("ferrum-kernels 0.7.7 src/stacked_expert.rs",
 * gemv_moe_id):
 * out[i, :] = a[i*src1_stride : i*src1_stride + n_cols] . dequant(W[ids[i]])^T,
 * i in [0, n_selected).  ids: device int32[n_selected].  out: [n_selected,
 * n_rows] in out_dtype (a_dtype or QMM_F32).  A pair whose id is outside
 * [0, num_experts) gets a zero row and sets QMM_ERR_BAD_EXPERT_ID in
 * *d_status. */
qmm_status qmm_moe_gemv_id(const void* a, qmm_dtype a_dtype, const int32_t* ids,
                           int64_t n_selected, int64_t src1_stride, const qmm_expert_stack* w,
                           void* out, qmm_dtype out_dtype, int32_t* d_status, void* stream);

/* Batched form (same page, gemv_moe_id_batched): ids is [m, top_k]
 * row-major; pair p in [0, m*top_k) reads
 * a[(p/top_k)*outer_stride + (p%top_k)*inner_stride : ... + n_cols] and
 * writes out[p, :]. */
qmm_status qmm_moe_gemv_id_batched(const void* a, qmm_dtype a_dtype, const int32_t* ids,
                                   int64_t m, int64_t top_k, int64_t outer_stride,
                                   int64_t inner_stride, const qmm_expert_stack* w, void* out,
                                   qmm_dtype out_dtype, int32_t* d_status, void* stream);

/* Fused gate/up (same page, gemv_moe_id_gate_up_silu):
 * silu_out[i, :] = SiLU(a . gate_e^T) * (a . up_e^T), e = ids[i], with
 * SiLU(g) = g / (1 + exp(-g)); every pair reads a[0 : n_cols] (the call has
 * no stride).  gate and up must have identical shapes and parameters
 * (QMM_ERR_INVALID_ARG otherwise).  Gate and up are computed in one pass. */
qmm_status qmm_moe_gemv_id_gate_up_silu(const void* a, qmm_dtype a_dtype, const int32_t* ids,
                                        int64_t n_selected, const qmm_expert_stack* gate,
                                        const qmm_expert_stack* up, void* silu_out,
                                        qmm_dtype out_dtype, int32_t* d_status, void* stream);

/* Batched fused form (same page, gemv_moe_id_gate_up_silu_batched): pair
 * offsets as in qmm_moe_gemv_id_batched.  The MoE errors for all four calls
 * are listed in the conventions above. */
qmm_status qmm_moe_gemv_id_gate_up_silu_batched(const void* a, qmm_dtype a_dtype,
                                                const int32_t* ids, int64_t m, int64_t top_k,
                                                int64_t outer_stride, int64_t inner_stride,
                                                const qmm_expert_stack* gate,
                                                const qmm_expert_stack* up, void* silu_out,
                                                qmm_dtype out_dtype, int32_t* d_status,
                                                void* stream);

/* ------------------------------------------------------------------------
 * MoE prefill GEMM: many tokens per expert ("ferrum-kernels 0.7.7
 * src/stacked_expert.rs", StackedExpertGgufLinear::gemm_moe_id and
 * gemm_moe_id_indirect, with the routing step of compute_ids_tpe_gpu).
 *
 *   out[p, :] = a[row(p), :] . dequant(W[ids[p]])^T,  p = token * top_k + slot
 *   row(p) = token when ne11 == 1 (a is [batch, K]: every slot of a token reads
 *            its row, as the gate and up projections do), p when ne11 == top_k
 *            (a is [batch * top_k, K]: one row per pair, as the down
 *            projection reads the per-slot activations).
 *
 * Two calls on one stream, no host round trip in between (the reason the
 * page's indirect variant exists): qmm_moe_compute_ids_tpe builds, on the
 * device, the tokens-per-expert counts, the pair indices grouped by expert
 * and the list of work blocks (<= 256 pairs of one expert each), together
 * with the page's 12-byte triple, in the caller's workspace; qmm_moe_gemm_id
 * reads that schedule on the device (its grid never depends on it).
 *
 * Workspace: qmm_moe_gemm_workspace_bytes(n_pairs, num_experts) bytes of
 * device memory, 4-byte aligned, owned by the caller and reused across calls;
 * int32 fields, in order, each padded to a multiple of 4 entries where noted:
 *   tpe[E]            pairs routed to expert e ("tokens per expert")
 *   off[E + 1]        exclusive prefix of tpe; off[E] = pairs with a valid id
 *   args[3]           {work blocks, largest tpe, experts with tpe > 0}
 *   (pad), pairs[n_pairs] (pad)   pair indices grouped by expert in expert
 *                     order (the order inside a group is unspecified);
 *                     pairs with an id outside [0, E) come last
 *   blk_e[nb] (pad), blk_s[nb] (pad)   expert and first entry of each block,
 *                     nb = ceil(n_pairs / 256) + E entries reserved
 * Optionally, from the next 256-byte boundary, room for the activation rows
 * gathered in pair-list order ([n_pairs, K] in a_dtype): a workspace of
 * qmm_moe_gemm_workspace_bytes_gathered(n_pairs, num_experts, K) bytes lets
 * qmm_moe_gemm_id copy each pair's row there once (one extra kernel) and
 * load every tile's rows as one contiguous TMA box, instead of gathering
 * them 4 rows per copy; same results.
 * A pair whose id is outside [0, E) gets a zero output row and sets
 * QMM_ERR_BAD_EXPERT_ID in *d_status (qmm_moe_compute_ids_tpe).
 * ------------------------------------------------------------------------ */

/* Workspace bytes for n_pairs pairs over num_experts experts (-1 when
 * n_pairs < 0, num_experts outside [1, 8192], or n_pairs > 2^30 - 1). */
int64_t qmm_moe_gemm_workspace_bytes(int64_t n_pairs, int64_t num_experts);

/* Workspace bytes that also hold the gathered activation rows of K = n_cols
 * 16-bit columns (-1 for the cases above or n_cols outside [1, 2^24]). */
int64_t qmm_moe_gemm_workspace_bytes_gathered(int64_t n_pairs, int64_t num_experts, int64_t n_cols);

/* Routing (compute_ids_tpe): ids is device int32[n_pairs] (the [batch, top_k]
 * routing table, row-major).  Writes the workspace fields above; one CTA.
 * Errors: INVALID_ARG (sizes, workspace_bytes too small), ALIGNMENT (ids,
 * workspace or d_status not 4-byte aligned), UNSUPPORTED (device), CUDA.
 * Device-side: QMM_ERR_BAD_EXPERT_ID in *d_status (may be NULL). */
qmm_status qmm_moe_compute_ids_tpe(const int32_t* ids, int64_t n_pairs, int64_t num_experts,
                                   void* workspace, int64_t workspace_bytes, int32_t* d_status,
                                   void* stream);

/* The expert-grouped GEMM over the schedule in `workspace` (written by
 * qmm_moe_compute_ids_tpe for the same n_pairs = batch * top_k and the same
 * number of experts, earlier on this stream).  a: [batch * ne11, K] in a_dtype
 * (bf16 or f16, equal to w->sdtype), K = w->n_cols; out: [batch * top_k,
 * w->n_rows] in out_dtype (a_dtype or f32), row p for pair p.  tcgen05 tensor
 * cores, fp32 accumulate, the dequantized weights rounded once to a_dtype.
 * Errors: INVALID_ARG (shapes, ne11 not 1 or top_k, workspace too small),
 * DTYPE, UNSUPPORTED (f32 activations, device), ALIGNMENT (a and out
 * 16-byte aligned, workspace 4-byte aligned), CUDA.  A device-side timeout
 * writes the affected tiles as NaN.  The call writes the workspace only in
 * the gathered-rows region, when the workspace has one. */
qmm_status qmm_moe_gemm_id(const void* a, qmm_dtype a_dtype, int64_t batch, int64_t top_k,
                           int64_t ne11, void* workspace, int64_t workspace_bytes,
                           const qmm_expert_stack* w, void* out, qmm_dtype out_dtype,
                           void* stream);

/* Allocation-free MoE prefill GEMM: routing and GEMM of qmm_moe_compute_ids_tpe
 * + qmm_moe_gemm_id in one call, with the routing schedule kept in a fixed
 * scratch array inside this library instead of a caller workspace.  The pages
 * have no counterpart; it serves callers that cannot provide device memory:
 * an operator or plugin interface that hands the op only its inputs and
 * outputs, or a latency-critical path where cudaMalloc (which may
 * synchronize the device) is not allowed.
 * Same arguments and results as the two calls (ids: device int32[batch *
 * top_k]; out: [batch * top_k, w->n_rows]), the same errors, plus
 * QMM_ERR_UNSUPPORTED when batch * top_k > 16384 or w->num_experts > 256 (the
 * scratch's capacity).  The scratch (about 70 KB) is held by every GPU that
 * loads the library until the process exits.  The first call on a device
 * looks up the scratch's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.  Every
 * call shares the one scratch array of its device: calls that overlap on the
 * GPU (on different streams, or in different threads) race and must be
 * serialized by the caller.  Each call rewrites all of the scratch it reads.
 * Allocates nothing. */
qmm_status qmm_moe_gemm_id_noalloc(const void* a, qmm_dtype a_dtype, const int32_t* ids,
                                   int64_t batch, int64_t top_k, int64_t ne11,
                                   const qmm_expert_stack* w, void* out, qmm_dtype out_dtype,
                                   int32_t* d_status, void* stream);

/* Diagnostic of the bounded device-side waits (not a step of the method).
 * Every TMA-fed kernel here waits on shared-memory mbarriers with a poll
 * limit and reports QMM_ERR_TIMEOUT instead of hanging when a wait gives up.
 * This call runs one tiny kernel that waits on a barrier nothing arrives on:
 *   d_result[0] = 1 if a wait on the already-completed phase returned at once,
 *   d_result[1] = 1 if the wait on the pending phase completed (expected 0:
 *                 it gives up after `spins` polls and ORs QMM_ERR_TIMEOUT into
 *                 *d_status),
 *   d_result[2] = 1 if the abortable wait completed with the abort flag
 *                 raised (expected 0).
 * d_result: device int32[3]; d_status: device int32, caller-zeroed; both
 * 4-byte aligned and required.  spins in [1, 2^22] (QMM_ERR_INVALID_ARG
 * otherwise).  Touches no memory but these two buffers and its own shared
 * memory; no copy is ever in flight.  Errors: INVALID_ARG, ALIGNMENT,
 * UNSUPPORTED (device), CUDA. */
qmm_status qmm_selftest_bounded_wait(uint32_t spins, int32_t* d_result, int32_t* d_status,
                                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QMM_H_ */
