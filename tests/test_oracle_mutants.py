"""Planted mistakes in the oracle must fail its pins (no GPU).

Each case copies ``oracle/qmm_oracle.c``, plants one plausible mistake (a
dropped term, a wrong sign, index or rounding rule, a transposed operand),
compiles the copy with the oracle's own flags, swaps it in for the real
library and runs the pins named beside it: at least one of them must fail.
A control compiles the unchanged source the same way and runs every pin the
cases use, so a harness fault cannot pass for a caught mistake.

The mistakes live only in temporary copies; the committed oracle is never
changed.
"""
import os

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "qmm_oracle.c")


def P(fn, **kw):
    return (fn, kw)


# (name, original text, planted text, pins that must catch it)
MUTANTS = [
    # scalar conversions
    ("bf16 rounding ties away from zero",
     "u += 0x7fffu + keep_lsb;", "u += 0x8000u;",
     [P(pins.test_bf16_conversion_matches_torch)]),
    ("f16 subnormal quantum off by a factor two",
     "nearbyint(a * 16777216.0)", "nearbyint(a * 8388608.0)",
     [P(pins.test_f16_conversion_matches_numpy)]),
    ("f16 exponent bias 14",
     "((E + 15) << 10)", "((E + 14) << 10)",
     [P(pins.test_f16_conversion_matches_numpy)]),
    # packing and unpacking
    ("dropped spill into the next word",
     "if (sh + bits > 32) words[wi + 1] |= q >> (32 - sh);", "",
     [P(pins.test_pack_matches_bigint_bitstream, bits=3),
      P(pins.test_cross_word_codes_straddle, bits=3, straddlers=[10, 21])]),
    ("spill shifted by the wrong amount",
     "words[wi + 1] |= q >> (32 - sh);", "words[wi + 1] |= q >> (31 - sh);",
     [P(pins.test_pack_matches_bigint_bitstream, bits=6)]),
    ("integral lanes read MSB-first",
     "return (w >> (lane * bits)) & ((1u << bits) - 1u);",
     "return (w >> ((lpu - 1 - lane) * bits)) & ((1u << bits) - 1u);",
     [P(pins.test_pack_matches_bigint_bitstream, bits=4)]),
    ("cross-word unpacker ignores the next word",
     "uint64_t both = cur | (nxt << 32);", "uint64_t both = cur | (nxt << 0 & 0);",
     [P(pins.test_pack_matches_bigint_bitstream, bits=3)]),
    # quantize
    ("scale divides by 2^b instead of 2^b - 1",
     "float scale_f = (mx - mn) / qmax;", "float scale_f = (mx - mn) / (qmax + 1.0f);",
     [P(pins.test_exact_grid_round_trip, bits=4, gs=64, sdt="f32"),
      P(pins.test_tie_rounds_half_away_from_zero)]),
    ("ties rounded to even",
     "float q = roundf(t);", "float q = rintf(t);",
     [P(pins.test_tie_rounds_half_away_from_zero)]),
    ("codes truncated instead of rounded",
     "float q = roundf(t);", "float q = floorf(t);",
     [P(pins.test_round_trip_bound_f32_storage, bits=4, gs=64)]),
    ("codes computed against the unrounded scale",
     "float t = (v - b) / s;", "float t = (v - b) / scale_f;",
     [P(pins.test_codes_are_nearest_on_the_stored_grid, bits=8, sdt="bf16"),
      P(pins.test_codes_are_nearest_on_the_stored_grid, bits=4, sdt="bf16")]),
    ("no clamp at the top code",
     "if (q > qmax) q = qmax;", "",
     [P(pins.test_codes_are_nearest_on_the_stored_grid, bits=8, sdt="bf16")]),
    ("no floor on the scale of a constant group",
     "if (scale_f < FLT_EPSILON) scale_f = FLT_EPSILON;", "",
     [P(pins.test_constant_group_is_exact)]),
    ("negative zero bias kept",
     "mn + 0.0f);", "mn);",
     [P(pins.test_constant_group_is_exact)]),
    ("group max taken as the bias",
     "float b = store_f(biases, s_dtype, r * G + g, mn + 0.0f);",
     "float b = store_f(biases, s_dtype, r * G + g, mx + 0.0f);",
     [P(pins.test_exact_grid_round_trip, bits=2, gs=32, sdt="f32")]),
    # dequantize
    ("bias subtracted",
     "return fmaf((float)q, s, b);", "return fmaf((float)q, s, -b);",
     [P(pins.test_dequant_exact_rational, bits=4, sdt="f32"),
      P(pins.test_exact_grid_round_trip, bits=4, gs=32, sdt="f32")]),
    ("two roundings instead of one fma",
     "return fmaf((float)q, s, b);", "return (float)q * s + b;",
     [P(pins.test_dequant_exact_rational, bits=8, sdt="bf16"),
      P(pins.test_dequant_exact_rational, bits=8, sdt="f32")]),
    ("group index wraps over the groups of a row",
     "int64_t g = i / gs;", "int64_t g = i % G;",
     [P(pins.test_dequant_exact_rational, bits=4, sdt="f32")]),
    # matmul
    ("x read transposed",
     "acc += (double)load_f(x, x_dtype, m * K + k) * (double)wcol[k];",
     "acc += (double)load_f(x, x_dtype, k * M + m) * (double)wcol[k];",
     [P(pins.test_matmul_brute_force_exact, bits=4, transpose=True)]),
    ("fp32 accumulator",
     "    for (int64_t m = 0; m < M; ++m) {\n      double acc = 0.0;",
     "    for (int64_t m = 0; m < M; ++m) {\n      float acc = 0.0f;",
     [P(pins.test_iota_example_quantized_matmul),
      P(pins.test_matmul_brute_force_exact, bits=8, transpose=True)]),
    ("transpose=0 reads the weights along the wrong axis",
     "wcol[k] = dequant_one(packed + k * wpr, wpr, scales, biases, s_dtype, k, G, gs, bits, n);",
     "wcol[k] = dequant_one(packed + n * wpr, wpr, scales, biases, s_dtype, n, G, gs, bits, k);",
     [P(pins.test_matmul_orientations_agree)]),
    # MoE
    ("pair offset ignores src1_stride",
     "expert_row_dot(st, e, n, a, a_dtype, i * src1_stride);",
     "expert_row_dot(st, e, n, a, a_dtype, 0);",
     [P(pins.test_moe_gemv_id_equals_per_pair_loop)]),
    ("batched offset swaps outer and inner",
     "int64_t off = (p / top_k) * outer + (p % top_k) * inner;\n    for (int64_t n = 0; n < st->n_rows; ++n) {",
     "int64_t off = (p % top_k) * outer + (p / top_k) * inner;\n    for (int64_t n = 0; n < st->n_rows; ++n) {",
     [P(pins.test_moe_batched_offsets_follow_the_page_formula)]),
    ("SiLU with the sign of the exponent flipped",
     "return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));",
     [P(pins.test_moe_gate_up_silu_closed_form)]),
    ("SiLU applied to up instead of gate",
     "out[i * gate->n_rows + n] = silu(g) * u;", "out[i * gate->n_rows + n] = g * silu(u);",
     [P(pins.test_moe_gate_up_silu_closed_form)]),
    ("bad expert id not reported",
     "        out[i * st->n_rows + n] = 0.0;\n        rc = ORC_ERR_ID;",
     "        out[i * st->n_rows + n] = 0.0;",
     [P(pins.test_moe_bad_id_reports_and_zero_fills)]),
    ("batched bad expert id not reported",
     "        out[p * st->n_rows + n] = 0.0;\n        rc = ORC_ERR_ID;",
     "        out[p * st->n_rows + n] = 0.0;",
     [P(pins.test_moe_bad_id_reports_and_zero_fills)]),
    ("fused bad expert id not reported",
     "        out[i * gate->n_rows + n] = 0.0;\n        rc = ORC_ERR_ID;",
     "        out[i * gate->n_rows + n] = 0.0;",
     [P(pins.test_moe_bad_id_reports_and_zero_fills)]),
    ("fused batched offset swaps outer and inner",
     "int64_t off = (p / top_k) * outer + (p % top_k) * inner;\n    for (int64_t n = 0; n < gate->n_rows; ++n) {",
     "int64_t off = (p % top_k) * outer + (p / top_k) * inner;\n    for (int64_t n = 0; n < gate->n_rows; ++n) {",
     [P(pins.test_moe_gate_up_silu_closed_form)]),
    # the single-element form used by the sampled full-size checks
    ("sampled element drops the first term",
     "  for (int64_t k = 0; k < K; ++k) {\n    float wv = transpose",
     "  for (int64_t k = 1; k < K; ++k) {\n    float wv = transpose",
     [P(pins.test_matmul_brute_force_exact, bits=4, transpose=True)]),
    # microscaled modes
    ("E2M1 sign bit ignored",
     "  return s ? -mag : mag;\n}\n\n/* FP8-E8M0", "  return mag;\n}\n\n/* FP8-E8M0",
     [P(pins.test_fp4_e2m1_matches_the_printed_table)]),
    ("E2M1 exponent bias 0",
     "ldexpf(1.0f + 0.5f * (float)m, e - 1)", "ldexpf(1.0f + 0.5f * (float)m, e)",
     [P(pins.test_fp4_e2m1_matches_the_printed_table)]),
    ("E8M0 bias 128",
     "ldexpf(1.0f, (int)(s & 0xff) - 127)", "ldexpf(1.0f, (int)(s & 0xff) - 128)",
     [P(pins.test_e8m0_is_two_to_the_byte_minus_127)]),
    ("E4M3 exponent shifted by 8",
     "(uint16_t)((b & 0x7f) << 7)", "(uint16_t)((b & 0x7f) << 8)",
     [P(pins.test_fp8_e4m3_matches_the_format_and_the_page)]),
    ("nvfp4 scales read as E8M0",
     "return mode == ORC_MODE_NVFP4 ? orc_fp8_e4m3(sbyte) : orc_e8m0(sbyte);",
     "return orc_e8m0(sbyte);",
     [P(pins.test_dequant_mx_exact_rational, mode=oracle.MODE_NVFP4)]),
    ("mxfp8 lanes decoded as E2M1",
     "return mode == ORC_MODE_MXFP8 ? orc_fp8_e4m3(code) : orc_fp4_e2m1(code);",
     "return orc_fp4_e2m1(code & 15);",
     [P(pins.test_dequant_mx_exact_rational, mode=oracle.MODE_MXFP8)]),
    ("nvfp4 group of 32",
     "case ORC_MODE_NVFP4: *bits = 4; *gs = 16; return 1;", "case ORC_MODE_NVFP4: *bits = 4; *gs = 32; return 1;",
     [P(pins.test_dequant_mx_exact_rational, mode=oracle.MODE_NVFP4)]),
    ("microscaled matmul drops the last term",
     "for (int64_t kk = 0; kk < K; ++kk) sum +=", "for (int64_t kk = 0; kk + 1 < K; ++kk) sum +=",
     [P(pins.test_matmul_mx_brute_force, mode=oracle.MODE_MXFP4)]),
    # per-tensor dynamic int8
    ("dynamic int8 offset 127",
     "float t = roundf((load_f(w, w_dtype, i) - mn) / scale) - 128.0f;",
     "float t = roundf((load_f(w, w_dtype, i) - mn) / scale) - 127.0f;",
     [P(pins.test_dynamic_int8_page_round_trip)]),
    ("dynamic int8 dequant adds the input minimum twice",
     "return scaled + params[2];", "return scaled + 2.0f * params[2];",
     [P(pins.test_dynamic_int8_dequant_exact_rational)]),
    ("dynamic int8 divides by 256",
     "float scale = (params[3] - params[2]) / 255.0f;", "float scale = (params[3] - params[2]) / 256.0f;",
     [P(pins.test_dynamic_int8_dequant_exact_rational), P(pins.test_dynamic_int8_page_round_trip)]),
    ("dynamic int8 without the epsilon floor",
     "if (!(scale >= FLT_EPSILON)) scale = FLT_EPSILON;", "",
     [P(pins.test_dynamic_int8_constant_tensor)]),
    ("dynamic int8 codes truncated",
     "float t = roundf((load_f(w, w_dtype, i) - mn) / scale) - 128.0f;",
     "float t = floorf((load_f(w, w_dtype, i) - mn) / scale) - 128.0f;",
     [P(pins.test_dynamic_int8_codes_are_nearest)]),
    ("dynamic int8 matmul reads the weight transposed",
     "(double)dyn8_one(q[nn * K + k], params);", "(double)dyn8_one(q[k * N + nn], params);",
     [P(pins.test_dynamic_int8_matmul_brute_force)]),
]


def _bind_source(text, tmp_path, name):
    src = tmp_path / f"{name}.c"
    src.write_text(text)
    return oracle.bind(oracle.compile_oracle(str(src), str(tmp_path / f"lib{name}.so")))


def _fails(fn, kw):
    try:
        fn(**kw)
    except AssertionError:
        return True
    return False


def test_control_unchanged_source_passes_every_pin(tmp_path, monkeypatch):
    monkeypatch.setattr(oracle, "_lib", _bind_source(open(SRC).read(), tmp_path, "control"))
    seen = set()
    for _, _, _, checks in MUTANTS:
        for fn, kw in checks:
            key = (fn.__name__, tuple(sorted((k, str(v)) for k, v in kw.items())))
            if key not in seen:
                seen.add(key)
                assert not _fails(fn, kw), f"{fn.__name__}{kw} fails on the unchanged oracle"


@pytest.mark.parametrize("name,orig,planted,checks", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(name, orig, planted, checks, tmp_path, monkeypatch):
    text = open(SRC).read()
    assert text.count(orig) == 1, f"mutation site for '{name}' is not unique in the oracle"
    monkeypatch.setattr(oracle, "_lib", _bind_source(text.replace(orig, planted), tmp_path, "m"))
    caught = [fn.__name__ for fn, kw in checks if _fails(fn, kw)]
    assert caught, f"no pin caught the planted mistake '{name}'"
