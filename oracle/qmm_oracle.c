/*
 * qmm_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * weight-only quantized matmul and its MoE indirect-dispatch variants.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no header, helper or table with the
 * CUDA path.
 *
 * Sources of the definitions (web pages, cited by title and section):
 *   [emily]  "emily 0.5.1 lib/emily/quantization.ex" -- quantized_matmul/2
 *            (x . to_dense(qw)^T), dequantize_defn/1 (lane i read at bit
 *            i*bits of the u32 stream, masked; w = lane*scale[g] + bias[g],
 *            g = i div group_size along the last axis), unpack_integral_lanes,
 *            unpack_cross_word_lanes, build_word_indices (clamped next word).
 *   [mlex]   "mlex 0.1.3 src/quant.rs" -- quantize_dynamic_int8: min/max
 *            quantizer, scale floored at f32::EPSILON, round() = half away
 *            from zero.  Used here as the model for the per-group affine
 *            quantizer (whose own body is not printed on any page), and
 *            written out itself (quantize_dynamic_int8,
 *            dequantize_dynamic_int8 with DynamicRangeParams) for the
 *            per-tensor int8 scheme.
 *   [ferrum] "ferrum-kernels 0.7.7 src/stacked_expert.rs" -- gemv_moe_id,
 *            gemv_moe_id_batched, gemv_moe_id_gate_up_silu(_batched).
 *
 * Floating point: compiled with -ffp-contract=off so every a*b+c in this
 * file is two roundings unless written as fmaf(); x86-64 SSE arithmetic has
 * no excess precision.
 *
 * Parity pins: every function here is pinned by tests/test_oracle_pins.py
 * (exact-rational recomputation, big-integer bitstreams, library dtype
 * conversions, closed forms); tests/test_oracle_mutants.py checks that
 * planted mistakes in a copy of this file fail those pins.  The accumulation
 * order of the GPU kernels is the only thing left "parity unpinned"
 * (tolerance only).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* dtype codes of this oracle (its own numbering; matches the order in which
 * the Python wrapper passes them) */
enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2 };

enum {
  ORC_OK = 0,
  ORC_ERR_ARG = 1,
  ORC_ERR_ID = 7
};

/* ------------------------------------------------------------------------ */
/* scalar conversions, written from the IEEE-754 binary16 / bfloat16 formats */
/* ------------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t h) {
  /* bfloat16 is the top half of a binary32 */
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

float orc_f16_to_f32(uint16_t h) {
  /* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits */
  int sign = (h >> 15) & 1;
  int ex = (h >> 10) & 0x1f;
  int man = h & 0x3ff;
  double v;
  if (ex == 0)
    v = ldexp((double)man, -24); /* subnormal: man * 2^-24 */
  else if (ex == 31)
    v = man ? NAN : INFINITY;
  else
    v = ldexp((double)(man | 0x400), ex - 25); /* (1024+man) * 2^(ex-15-10) */
  return (float)(sign ? -v : v);
}

uint16_t orc_f32_to_bf16(float f) {
  /* round to nearest, ties to even, on the 16 dropped bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t keep_lsb = (u >> 16) & 1u;
  u += 0x7fffu + keep_lsb;
  return (uint16_t)(u >> 16);
}

uint16_t orc_f32_to_f16(float f) {
  /* round to nearest, ties to even (nearbyint under the default mode) */
  uint32_t u;
  memcpy(&u, &f, 4);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
  double a = fabs((double)f);
  if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u); /* >= midpoint(65504, 2^16) */
  if (a < ldexp(1.0, -14)) {
    /* subnormal range: quantum 2^-24; 1024 quanta encodes the smallest normal */
    double r = nearbyint(a * 16777216.0);
    return (uint16_t)(sign | (uint16_t)r);
  }
  int e;
  (void)frexp(a, &e);         /* a = m * 2^e, m in [0.5, 1) */
  int E = e - 1;              /* a in [2^E, 2^(E+1)) */
  double q = ldexp(a, 10 - E); /* in [1024, 2048) */
  double r = nearbyint(q);
  if (r == 2048.0) {
    r = 1024.0;
    E += 1;
  }
  if (E > 15) return (uint16_t)(sign | 0x7c00u);
  return (uint16_t)(sign | (uint16_t)(((E + 15) << 10) | ((int)r - 1024)));
}

static float load_f(const void* p, int dtype, int64_t i) {
  switch (dtype) {
    case ORC_F32: return ((const float*)p)[i];
    case ORC_F16: return orc_f16_to_f32(((const uint16_t*)p)[i]);
    default: return orc_bf16_to_f32(((const uint16_t*)p)[i]);
  }
}

/* store v in `dtype` (one RNE rounding) and return the stored value widened */
static float store_f(void* p, int dtype, int64_t i, float v) {
  switch (dtype) {
    case ORC_F32: ((float*)p)[i] = v; return v;
    case ORC_F16: {
      uint16_t h = orc_f32_to_f16(v);
      ((uint16_t*)p)[i] = h;
      return orc_f16_to_f32(h);
    }
    default: {
      uint16_t h = orc_f32_to_bf16(v);
      ((uint16_t*)p)[i] = h;
      return orc_bf16_to_f32(h);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* parameter checks                                                          */
/* ------------------------------------------------------------------------ */

static int bits_ok(int bits) {
  return bits == 2 || bits == 3 || bits == 4 || bits == 6 || bits == 8;
}

static int shape_ok(int64_t cols, int gs, int bits) {
  if (!bits_ok(bits)) return 0;
  if (gs != 32 && gs != 64 && gs != 128) return 0;
  if (cols <= 0 || cols % gs) return 0;
  if ((cols * bits) % 32) return 0; /* [emily] build_word_indices invariant */
  return 1;
}

int64_t orc_words_per_row(int64_t cols, int bits) { return cols * bits / 32; }

/* ------------------------------------------------------------------------ */
/* packing: LSB-first bitstream along the row                                */
/* ------------------------------------------------------------------------ */

/* Code j of a row occupies stream bits [j*bits, (j+1)*bits): the low part
 * goes to word (j*bits)>>5 at shift (j*bits)&31, any spill to the next word. */
void orc_pack_row(const uint8_t* codes, int64_t cols, int bits, uint32_t* words) {
  int64_t nw = orc_words_per_row(cols, bits);
  for (int64_t w = 0; w < nw; ++w) words[w] = 0;
  for (int64_t j = 0; j < cols; ++j) {
    int64_t p = j * bits;
    int64_t wi = p >> 5;
    int sh = (int)(p & 31);
    uint32_t q = codes[j];
    words[wi] |= q << sh;
    if (sh + bits > 32) words[wi + 1] |= q >> (32 - sh);
  }
}

/* unpacker 1 ([emily] unpack_integral_lanes): bits in {2,4,8};
 * word i / lanes_per_word, shifted by lane*bits, masked */
uint32_t orc_code_integral(const uint32_t* row, int bits, int64_t i) {
  int lpu = 32 / bits;
  uint32_t w = row[i / lpu];
  int lane = (int)(i % lpu);
  return (w >> (lane * bits)) & ((1u << bits) - 1u);
}

/* unpacker 2 ([emily] unpack_cross_word_lanes): the word holding bit i*bits
 * and the next one (clamped to the last word of the row) read as one u64,
 * shifted by (i*bits) mod 32, masked */
uint32_t orc_code_u64(const uint32_t* row, int64_t words_per_row, int bits, int64_t i) {
  int64_t wi = (i * bits) / 32;
  int64_t nx = wi + 1 < words_per_row - 1 ? wi + 1 : words_per_row - 1;
  uint64_t cur = row[wi];
  uint64_t nxt = row[nx];
  uint64_t both = cur | (nxt << 32);
  return (uint32_t)((both >> ((i * bits) % 32)) & ((1ull << bits) - 1ull));
}

/* the page picks the integral path when 32 is a multiple of bits */
static uint32_t code_at(const uint32_t* row, int64_t wpr, int bits, int64_t i) {
  if (32 % bits == 0) return orc_code_integral(row, bits, i);
  return orc_code_u64(row, wpr, bits, i);
}

/* ------------------------------------------------------------------------ */
/* quantize: per (row, group) min/max affine                                 */
/* ------------------------------------------------------------------------ */

/* For each group of `gs` consecutive columns of a row:
 *   mn, mx   = min, max of the group (fp32 compares)
 *   scale_f  = (mx - mn) / (2^bits - 1)         one fp32 rounding
 *   scale_f  = max(scale_f, FLT_EPSILON)        ([mlex] EPSILON floor)
 *   s        = scale_f rounded to s_dtype       (RNE)
 *   bias     = (mn + 0) rounded to s_dtype      (+0 turns -0 into +0)
 *   q        = clamp(roundf((w - bias) / s), 0, 2^bits - 1)
 *              w - bias and / each one fp32 rounding, against the STORED
 *              s and bias; roundf = half away from zero ([mlex] round()).
 * Codes are then packed LSB-first.  Rows [r0, r1) only. */
int orc_quantize(const void* w, int w_dtype, int64_t rows, int64_t cols, int gs, int bits,
                 int s_dtype, uint32_t* packed, void* scales, void* biases, int64_t r0,
                 int64_t r1) {
  if (!shape_ok(cols, gs, bits) || rows < 0) return ORC_ERR_ARG;
  int64_t wpr = orc_words_per_row(cols, bits);
  int64_t G = cols / gs;
  float qmax = (float)((1 << bits) - 1);
  uint8_t* codes = (uint8_t*)malloc((size_t)cols);
  if (!codes) return ORC_ERR_ARG;
  for (int64_t r = r0; r < r1; ++r) {
    for (int64_t g = 0; g < G; ++g) {
      int64_t base = r * cols + g * gs;
      float mn = load_f(w, w_dtype, base);
      float mx = mn;
      for (int i = 1; i < gs; ++i) {
        float v = load_f(w, w_dtype, base + i);
        if (v < mn) mn = v;
        if (v > mx) mx = v;
      }
      float scale_f = (mx - mn) / qmax;
      if (scale_f < FLT_EPSILON) scale_f = FLT_EPSILON;
      float s = store_f(scales, s_dtype, r * G + g, scale_f);
      float b = store_f(biases, s_dtype, r * G + g, mn + 0.0f);
      for (int i = 0; i < gs; ++i) {
        float v = load_f(w, w_dtype, base + i);
        float t = (v - b) / s;
        float q = roundf(t);
        if (q < 0.0f) q = 0.0f;
        if (q > qmax) q = qmax;
        codes[g * gs + i] = (uint8_t)q;
      }
    }
    orc_pack_row(codes, cols, bits, packed + r * wpr);
  }
  free(codes);
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* dequantize                                                                */
/* ------------------------------------------------------------------------ */

/* w_hat = fmaf((float)q, s, bias): one fp32 rounding; stored in out_dtype
 * with one RNE rounding (none for fp32).  The page's Nx graph computes
 * q*s + b in the scales dtype (two roundings for bf16); this oracle follows
 * the single-rounding fmaf definition instead. */
static float dequant_one(const uint32_t* row, int64_t wpr, const void* scales,
                         const void* biases, int s_dtype, int64_t r, int64_t G, int gs,
                         int bits, int64_t i) {
  uint32_t q = code_at(row, wpr, bits, i);
  int64_t g = i / gs;
  float s = load_f(scales, s_dtype, r * G + g);
  float b = load_f(biases, s_dtype, r * G + g);
  return fmaf((float)q, s, b);
}

int orc_dequantize(const uint32_t* packed, const void* scales, const void* biases, int s_dtype,
                   int64_t rows, int64_t cols, int gs, int bits, void* out, int out_dtype,
                   int64_t r0, int64_t r1) {
  if (!shape_ok(cols, gs, bits) || rows < 0) return ORC_ERR_ARG;
  int64_t wpr = orc_words_per_row(cols, bits);
  int64_t G = cols / gs;
  for (int64_t r = r0; r < r1; ++r) {
    const uint32_t* row = packed + r * wpr;
    for (int64_t i = 0; i < cols; ++i) {
      float v = dequant_one(row, wpr, scales, biases, s_dtype, r, G, gs, bits, i);
      store_f(out, out_dtype, r * cols + i, v);
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* matmul: y = x . dequant(W)^T  (transpose = 1)  or  x . dequant(W)  (0)     */
/* ------------------------------------------------------------------------ */

/* transpose = 1: packed is [N, K] quantized along K; y[m][n] = sum_k x[m][k] w[n][k]
 * transpose = 0: packed is [K, N] quantized along N; y[m][n] = sum_k x[m][k] w[k][n]
 * Products and sums in fp64, k increasing.  Output columns [n0, n1) only. */
int orc_matmul(const void* x, int x_dtype, int64_t M, int64_t K, const uint32_t* packed,
               const void* scales, const void* biases, int s_dtype, int64_t N, int gs,
               int bits, int transpose, double* y, int64_t n0, int64_t n1) {
  int64_t qcols = transpose ? K : N; /* quantized axis */
  if (!shape_ok(qcols, gs, bits) || M < 0 || K <= 0 || N <= 0) return ORC_ERR_ARG;
  int64_t wpr = orc_words_per_row(qcols, bits);
  int64_t G = qcols / gs;
  float* wcol = (float*)malloc(sizeof(float) * (size_t)K);
  if (!wcol) return ORC_ERR_ARG;
  for (int64_t n = n0; n < n1; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      if (transpose)
        wcol[k] = dequant_one(packed + n * wpr, wpr, scales, biases, s_dtype, n, G, gs, bits, k);
      else
        wcol[k] = dequant_one(packed + k * wpr, wpr, scales, biases, s_dtype, k, G, gs, bits, n);
    }
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += (double)load_f(x, x_dtype, m * K + k) * (double)wcol[k];
      y[m * N + n] = acc;
    }
  }
  free(wcol);
  return ORC_OK;
}

/* one output element y[m][n] (for sampled checks at full size) */
double orc_matmul_element(const void* x, int x_dtype, int64_t M, int64_t K,
                          const uint32_t* packed, const void* scales, const void* biases,
                          int s_dtype, int64_t N, int gs, int bits, int transpose, int64_t m,
                          int64_t n) {
  int64_t qcols = transpose ? K : N;
  int64_t wpr = orc_words_per_row(qcols, bits);
  int64_t G = qcols / gs;
  (void)M;
  double acc = 0.0;
  for (int64_t k = 0; k < K; ++k) {
    float wv = transpose
                   ? dequant_one(packed + n * wpr, wpr, scales, biases, s_dtype, n, G, gs, bits, k)
                   : dequant_one(packed + k * wpr, wpr, scales, biases, s_dtype, k, G, gs, bits, n);
    acc += (double)load_f(x, x_dtype, m * K + k) * (double)wv;
  }
  return acc;
}

/* ------------------------------------------------------------------------ */
/* MoE stacked experts ([ferrum] StackedExpertGgufLinear)                    */
/* ------------------------------------------------------------------------ */

/* Expert e of a stack occupies rows [e*n_rows, (e+1)*n_rows) of one packed
 * [E*n_rows, n_cols*bits/32] u32 array and of the [E*n_rows, n_cols/gs]
 * scale and bias arrays (N experts stored contiguously). */
typedef struct {
  const uint32_t* packed;
  const void* scales;
  const void* biases;
  int s_dtype;
  int64_t num_experts, n_rows, n_cols;
  int gs, bits;
} orc_stack;

static int stack_ok(const orc_stack* st) {
  return st && st->num_experts > 0 && st->n_rows > 0 && shape_ok(st->n_cols, st->gs, st->bits);
}

/* dot(a[0:n_cols], w_hat_e[n, :]) in fp64 */
static double expert_row_dot(const orc_stack* st, int64_t e, int64_t n, const void* a,
                             int a_dtype, int64_t a_off) {
  int64_t wpr = orc_words_per_row(st->n_cols, st->bits);
  int64_t G = st->n_cols / st->gs;
  int64_t r = e * st->n_rows + n;
  const uint32_t* row = st->packed + r * wpr;
  double acc = 0.0;
  for (int64_t k = 0; k < st->n_cols; ++k) {
    float wv = dequant_one(row, wpr, st->scales, st->biases, st->s_dtype, r, G, st->gs,
                           st->bits, k);
    acc += (double)load_f(a, a_dtype, a_off + k) * (double)wv;
  }
  return acc;
}

/* out[i, :] = a[i*src1_stride : +n_cols] . w_hat[ids[i]]^T, pairs [i0, i1).
 * Returns ORC_ERR_ID (and leaves the pair's row zero) for ids outside [0, E). */
int orc_moe_gemv_id(const void* a, int a_dtype, const int32_t* ids, int64_t n_selected,
                    int64_t src1_stride, const orc_stack* st, double* out, int64_t i0,
                    int64_t i1) {
  if (!stack_ok(st) || n_selected < 0) return ORC_ERR_ARG;
  int rc = ORC_OK;
  for (int64_t i = i0; i < i1; ++i) {
    int64_t e = ids[i];
    for (int64_t n = 0; n < st->n_rows; ++n) {
      if (e < 0 || e >= st->num_experts) {
        out[i * st->n_rows + n] = 0.0;
        rc = ORC_ERR_ID;
        continue;
      }
      out[i * st->n_rows + n] = expert_row_dot(st, e, n, a, a_dtype, i * src1_stride);
    }
  }
  return rc;
}

/* pair p reads a[(p/top_k)*outer + (p%top_k)*inner]; ids is [m, top_k] */
int orc_moe_gemv_id_batched(const void* a, int a_dtype, const int32_t* ids, int64_t m,
                            int64_t top_k, int64_t outer, int64_t inner, const orc_stack* st,
                            double* out, int64_t p0, int64_t p1) {
  if (!stack_ok(st) || m < 0 || top_k <= 0) return ORC_ERR_ARG;
  int rc = ORC_OK;
  for (int64_t p = p0; p < p1; ++p) {
    int64_t e = ids[p];
    int64_t off = (p / top_k) * outer + (p % top_k) * inner;
    for (int64_t n = 0; n < st->n_rows; ++n) {
      if (e < 0 || e >= st->num_experts) {
        out[p * st->n_rows + n] = 0.0;
        rc = ORC_ERR_ID;
        continue;
      }
      out[p * st->n_rows + n] = expert_row_dot(st, e, n, a, a_dtype, off);
    }
  }
  return rc;
}

static int same_shape(const orc_stack* g, const orc_stack* u) {
  return g->num_experts == u->num_experts && g->n_rows == u->n_rows && g->n_cols == u->n_cols &&
         g->gs == u->gs && g->bits == u->bits && g->s_dtype == u->s_dtype;
}

/* SiLU(g) = g / (1 + exp(-g)) (textbook; the page only names it), in fp64 */
static double silu(double g) { return g / (1.0 + exp(-g)); }

/* silu_out[p, :] = SiLU(a_p . gate_e^T) * (a_p . up_e^T), e = ids[p].
 * Non-batched form: every pair reads a[0:n_cols] (offset 0). */
int orc_moe_gate_up_silu(const void* a, int a_dtype, const int32_t* ids, int64_t n_selected,
                         const orc_stack* gate, const orc_stack* up, double* out, int64_t i0,
                         int64_t i1) {
  if (!stack_ok(gate) || !stack_ok(up) || !same_shape(gate, up) || n_selected < 0)
    return ORC_ERR_ARG;
  int rc = ORC_OK;
  for (int64_t i = i0; i < i1; ++i) {
    int64_t e = ids[i];
    for (int64_t n = 0; n < gate->n_rows; ++n) {
      if (e < 0 || e >= gate->num_experts) {
        out[i * gate->n_rows + n] = 0.0;
        rc = ORC_ERR_ID;
        continue;
      }
      double g = expert_row_dot(gate, e, n, a, a_dtype, 0);
      double u = expert_row_dot(up, e, n, a, a_dtype, 0);
      out[i * gate->n_rows + n] = silu(g) * u;
    }
  }
  return rc;
}

int orc_moe_gate_up_silu_batched(const void* a, int a_dtype, const int32_t* ids, int64_t m,
                                 int64_t top_k, int64_t outer, int64_t inner,
                                 const orc_stack* gate, const orc_stack* up, double* out,
                                 int64_t p0, int64_t p1) {
  if (!stack_ok(gate) || !stack_ok(up) || !same_shape(gate, up) || m < 0 || top_k <= 0)
    return ORC_ERR_ARG;
  int rc = ORC_OK;
  for (int64_t p = p0; p < p1; ++p) {
    int64_t e = ids[p];
    int64_t off = (p / top_k) * outer + (p % top_k) * inner;
    for (int64_t n = 0; n < gate->n_rows; ++n) {
      if (e < 0 || e >= gate->num_experts) {
        out[p * gate->n_rows + n] = 0.0;
        rc = ORC_ERR_ID;
        continue;
      }
      double g = expert_row_dot(gate, e, n, a, a_dtype, off);
      double u = expert_row_dot(up, e, n, a, a_dtype, off);
      out[p * gate->n_rows + n] = silu(g) * u;
    }
  }
  return rc;
}

/* ------------------------------------------------------------------------ */
/* microscaled modes ([emily] dequantize_mxfp4_impl, dequantize_mxfp8_impl, */
/* dequantize_nvfp4_impl, fp4_lut, e8m0_lut, fp8_e4m3_lut; group sizes:      */
/* [emily] "one per group of 32 lanes" for mxfp4/mxfp8, [ollama]             */
/* quantizeParams {16, 4, "nvfp4"}, {32, 8, "mxfp8"})                        */
/* ------------------------------------------------------------------------ */

enum { ORC_MODE_AFFINE = 0, ORC_MODE_MXFP4 = 1, ORC_MODE_MXFP8 = 2, ORC_MODE_NVFP4 = 3 };

/* FP4-E2M1 lane: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa;
 * exponent 0 is the subnormal 0.5 * m, otherwise 2^(e-1) * (1 + m/2). */
float orc_fp4_e2m1(uint32_t c) {
  int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
  float mag = e == 0 ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
  return s ? -mag : mag;
}

/* FP8-E8M0 scale byte: 2^(s - 127) (s = 255 overflows fp32 to +inf) */
float orc_e8m0(uint32_t s) { return ldexpf(1.0f, (int)(s & 0xff) - 127); }

/* FP8-E4M3 byte as the page decodes it: the low 7 bits shifted left by 7
 * read as a binary16, times 256, then the sign of bit 7 (so 0x7F and 0xFF
 * are +-480 rather than NaN). */
float orc_fp8_e4m3(uint32_t b) {
  float mag = orc_f16_to_f32((uint16_t)((b & 0x7f) << 7)) * 256.0f;
  return (b & 0x80) ? -mag : mag;
}

/* bits and group size of a microscaled mode (0 for any other mode) */
int orc_mx_params(int mode, int* bits, int* gs) {
  switch (mode) {
    case ORC_MODE_MXFP4: *bits = 4; *gs = 32; return 1;
    case ORC_MODE_MXFP8: *bits = 8; *gs = 32; return 1;
    case ORC_MODE_NVFP4: *bits = 4; *gs = 16; return 1;
    default: return 0;
  }
}

static float mx_lane(int mode, uint32_t code) {
  return mode == ORC_MODE_MXFP8 ? orc_fp8_e4m3(code) : orc_fp4_e2m1(code);
}

static float mx_scale(int mode, uint8_t sbyte) {
  return mode == ORC_MODE_NVFP4 ? orc_fp8_e4m3(sbyte) : orc_e8m0(sbyte);
}

/* w_hat[r][i] = lane(q) * scale(s[r][i / gs]): one fp32 product (the page
 * multiplies the two table values in bf16; both tables' values and their
 * products are exact in bf16 for the scales the quantizers emit, so the fp32
 * product is the same number).  No bias. */
static float dequant_mx_one(const uint32_t* row, const uint8_t* scales, int mode, int bits, int gs,
                            int64_t r, int64_t G, int64_t i) {
  uint32_t q = orc_code_integral(row, bits, i);
  return mx_lane(mode, q) * mx_scale(mode, scales[r * G + i / gs]);
}

int orc_dequantize_mx(const uint32_t* packed, const uint8_t* scales, int mode, int64_t rows,
                      int64_t cols, void* out, int out_dtype, int64_t r0, int64_t r1) {
  int bits, gs;
  if (!orc_mx_params(mode, &bits, &gs) || rows < 0 || cols <= 0 || cols % gs) return ORC_ERR_ARG;
  int64_t wpr = orc_words_per_row(cols, bits);
  int64_t G = cols / gs;
  for (int64_t r = r0; r < r1; ++r)
    for (int64_t i = 0; i < cols; ++i)
      store_f(out, out_dtype, r * cols + i,
              dequant_mx_one(packed + r * wpr, scales, mode, bits, gs, r, G, i));
  return ORC_OK;
}

/* y[m][n] = sum_k x[m][k] * w_hat[n][k] (W is [N, K] quantized along K), in
 * fp64 with k increasing.  Output columns [n0, n1) only. */
int orc_matmul_mx(const void* x, int x_dtype, int64_t M, int64_t K, const uint32_t* packed,
                  const uint8_t* scales, int mode, int64_t N, double* y, int64_t n0, int64_t n1) {
  int bits, gs;
  if (!orc_mx_params(mode, &bits, &gs) || M < 0 || K <= 0 || N <= 0 || K % gs) return ORC_ERR_ARG;
  int64_t wpr = orc_words_per_row(K, bits);
  int64_t G = K / gs;
  float* wcol = (float*)malloc(sizeof(float) * (size_t)K);
  if (!wcol) return ORC_ERR_ARG;
  for (int64_t n = n0; n < n1; ++n) {
    for (int64_t k = 0; k < K; ++k) wcol[k] = dequant_mx_one(packed + n * wpr, scales, mode, bits, gs, n, G, k);
    for (int64_t m = 0; m < M; ++m) {
      double sum = 0.0;
      for (int64_t kk = 0; kk < K; ++kk) sum += (double)load_f(x, x_dtype, m * K + kk) * (double)wcol[kk];
      y[m * N + n] = sum;
    }
  }
  free(wcol);
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* per-tensor dynamic-range int8 ([mlex] quantize_dynamic_int8,             */
/* dequantize_dynamic_int8, DynamicRangeParams)                             */
/* ------------------------------------------------------------------------ */

/* params = {input_min, input_max, output_min, output_max} = {mn, mx, mn, mx}
 * with mn, mx the whole tensor's min and max: a fold that starts at +inf
 * (-inf) and takes fminf (fmaxf), which passes over NaN elements as the
 * page's f32::min / f32::max do;
 * scale = max((mx - mn) / 255, FLT_EPSILON);
 * q = clamp(round((w - mn) / scale) - 128, -128, 127), each of -, /, round
 * (half away from zero), -128 in fp32; a NaN t becomes code 0 (the page's
 * float-to-i8 cast). */
int orc_quantize_dynamic_int8(const void* w, int w_dtype, int64_t n, int8_t* q, float* params) {
  if (n <= 0) return ORC_ERR_ARG;
  float mn = INFINITY, mx = -INFINITY;
  for (int64_t i = 0; i < n; ++i) {
    float v = load_f(w, w_dtype, i);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  float scale = (mx - mn) / 255.0f;
  if (!(scale >= FLT_EPSILON)) scale = FLT_EPSILON; /* f32::max: a NaN side loses */
  for (int64_t i = 0; i < n; ++i) {
    float t = roundf((load_f(w, w_dtype, i) - mn) / scale) - 128.0f;
    if (t < -128.0f) t = -128.0f;
    if (t > 127.0f) t = 127.0f;
    q[i] = isnan(t) ? (int8_t)0 : (int8_t)t;
  }
  params[0] = mn;
  params[1] = mx;
  params[2] = mn;
  params[3] = mx;
  return ORC_OK;
}

/* w_hat = ((float)q + 128) * scale + output_min, scale = (output_max -
 * output_min) / 255: the page's three fp32 operations in its order (the sum
 * with 128 is exact; the product and the final sum round once each). */
static float dyn8_one(int8_t q, const float* params) {
  float scale = (params[3] - params[2]) / 255.0f;
  float shifted = (float)q + 128.0f;
  float scaled = shifted * scale;
  return scaled + params[2];
}

int orc_dequantize_dynamic_int8(const int8_t* q, int64_t n, const float* params, void* out, int out_dtype) {
  if (n < 0) return ORC_ERR_ARG;
  for (int64_t i = 0; i < n; ++i) store_f(out, out_dtype, i, dyn8_one(q[i], params));
  return ORC_OK;
}

/* y[m][n] = sum_k x[m][k] * w_hat[n][k] (W is [N, K] int8), fp64 sums with k
 * increasing.  Output columns [n0, n1) only. */
int orc_matmul_dynamic_int8(const void* x, int x_dtype, int64_t M, int64_t K, const int8_t* q,
                            const float* params, int64_t N, double* y, int64_t n0, int64_t n1) {
  if (M < 0 || K <= 0 || N <= 0) return ORC_ERR_ARG;
  for (int64_t nn = n0; nn < n1; ++nn)
    for (int64_t m = 0; m < M; ++m) {
      double dot = 0.0;
      for (int64_t k = 0; k < K; ++k)
        dot += (double)load_f(x, x_dtype, m * K + k) * (double)dyn8_one(q[nn * K + k], params);
      y[m * N + nn] = dot;
    }
  return ORC_OK;
}
