"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: library
dtype conversions, Python big-integer bitstreams, exact rational arithmetic,
closed forms, grid weights whose quantization is known in advance, and the
examples printed on the pages (tests/golden/pages_examples.json).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests import exact
from weight_only_quantized_qmm_b200 import workloads as wl

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_examples.json")))
BITS = GOLDEN["defn_supported_bits"]["value"]
GROUPS = [32, 64, 128]
DT = {"f32": oracle.F32, "f16": oracle.F16, "bf16": oracle.BF16}


def to_storage(t: torch.Tensor, dtype: str) -> np.ndarray:
    return wl.storage_numpy(t.to({"f32": torch.float32, "f16": torch.float16,
                                  "bf16": torch.bfloat16}[dtype]))


def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """storage form -> float64 via numpy/torch (library routines)"""
    if dtype == "f32":
        return a.astype(np.float64)
    if dtype == "f16":
        return a.view(np.float16).astype(np.float64)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ conversions
SPECIAL = [0.0, -0.0, 1.0, -1.0, 1e-8, 5.96e-8, 6.1e-5, 6.0e-5, 65504.0, 65519.0, 65520.0,
           70000.0, 3.0e38, 1.0 + 2.0**-8, 1.0 + 3 * 2.0**-9, 1.0 + 2.0**-11, 1.0 + 3 * 2.0**-12,
           2.0**-24, 2.0**-25, 3 * 2.0**-26, 1.17549435e-38, float("inf"), -float("inf")]


def test_bf16_conversion_matches_torch():
    rng = np.random.default_rng(1)
    vals = np.concatenate([np.array(SPECIAL, dtype=np.float32),
                           rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 4000)])
    ref = wl.storage_numpy(torch.from_numpy(vals).to(torch.bfloat16))
    got = np.array([oracle.f32_to_bf16(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(ref, got)
    back = np.array([oracle.bf16_to_f32(int(h)) for h in got], dtype=np.float32)
    assert np.array_equal(back, torch.from_numpy(vals).to(torch.bfloat16).float().numpy())


def test_f16_conversion_matches_numpy():
    rng = np.random.default_rng(2)
    vals = np.concatenate([np.array(SPECIAL, dtype=np.float32),
                           (rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 6, 4000)).astype(np.float32)])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f32_to_f16(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(ref, got)
    allbits = np.arange(0, 1 << 16, dtype=np.uint16)
    finite = np.isfinite(allbits.view(np.float16))
    back = np.array([oracle.f16_to_f32(int(h)) for h in allbits[finite]], dtype=np.float32)
    assert np.array_equal(back, allbits[finite].view(np.float16).astype(np.float32))


# ------------------------------------------------------------------ packing
@pytest.mark.parametrize("bits", BITS)
def test_pack_matches_bigint_bitstream(bits):
    rng = np.random.default_rng(bits)
    for cols in (32, 64, 96, 160, 512):
        if (cols * bits) % 32:
            continue
        codes = rng.integers(0, 1 << bits, cols).astype(np.uint8)
        words = oracle.pack_row(codes, bits)
        assert words.size == cols * bits // 32 == oracle.words_per_row(cols, bits)
        assert words.tolist() == exact.pack_bigint(codes.tolist(), bits)
        # unpacker 2 (u64 pair) on every width, unpacker 1 on the integral widths
        got2 = [oracle.code_u64(words, bits, i) for i in range(cols)]
        assert got2 == codes.tolist()
        if 32 % bits == 0:
            got1 = [oracle.code_integral(words, bits, i) for i in range(cols)]
            assert got1 == got2


@pytest.mark.parametrize("bits,straddlers", [(3, [10, 21]), (6, [5, 10, 21, 26])])
def test_cross_word_codes_straddle(bits, straddlers):
    """3-bit code 10 sits on bits 30..32 (words 0|1), code 21 on 63..65 (words 1|2)."""
    cols = 32 if bits == 3 else 32
    for j in straddlers:
        codes = np.zeros(cols, dtype=np.uint8)
        codes[j] = (1 << bits) - 1
        words = oracle.pack_row(codes, bits)
        lo = (j * bits) // 32
        assert words[lo] != 0 and words[lo + 1] != 0, "code must span two words"
        assert words.tolist() == exact.pack_bigint(codes.tolist(), bits)
        assert oracle.code_u64(words, bits, j) == (1 << bits) - 1


# ------------------------------------------------------------------ quantize / dequantize
def _grid_weight(bits, gs, rows, cols, rng, s_exp=-7):
    """W = bias + q*s exactly, with each group containing both 0 and 2^b-1."""
    s = 2.0 ** s_exp
    qmax = (1 << bits) - 1
    q = rng.integers(0, qmax + 1, (rows, cols))
    q[:, ::gs] = 0
    q[:, 1::gs] = qmax
    G = cols // gs
    c = rng.integers(-64, 64, (rows, G))
    bias = -c * s
    w = np.repeat(bias, gs, axis=1) + q * s
    return w.astype(np.float32), q, np.full((rows, G), s), bias


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("gs", GROUPS)
@pytest.mark.parametrize("sdt", ["f32", "bf16"])
def test_exact_grid_round_trip(bits, gs, sdt):
    rng = np.random.default_rng(bits * 1000 + gs)
    rows, cols = 6, 4 * gs
    w, q, s, b = _grid_weight(bits, gs, rows, cols, rng)
    packed, sc, bi = oracle.quantize(w, oracle.F32, gs, bits, DT[sdt])
    assert np.array_equal(widen(sc, sdt), s)
    assert np.array_equal(widen(bi, sdt), b)
    codes = np.array([exact.unpack_bigint(packed[r].tolist(), bits, cols) for r in range(rows)])
    assert np.array_equal(codes, q)
    deq = oracle.dequantize(packed, sc, bi, DT[sdt], cols, gs, bits, oracle.F32)
    assert np.array_equal(deq, w)


def _fraction_dequant(codes, s, b):
    """exact q*s + b, rounded once to fp32 (the fmaf definition)"""
    return exact.rf32(Fraction(int(codes)) * s + b)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("sdt", ["f32", "bf16", "f16"])
def test_dequant_exact_rational(bits, sdt):
    rng = np.random.default_rng(7 + bits)
    gs, rows, cols = 32, 3, 64
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    packed, sc, bi = oracle.quantize(w, oracle.F32, gs, bits, DT[sdt])
    out32 = oracle.dequantize(packed, sc, bi, DT[sdt], cols, gs, bits, oracle.F32)
    outbf = oracle.dequantize(packed, sc, bi, DT[sdt], cols, gs, bits, oracle.BF16)
    outh = oracle.dequantize(packed, sc, bi, DT[sdt], cols, gs, bits, oracle.F16)
    for r in range(rows):
        codes = exact.unpack_bigint(packed[r].tolist(), bits, cols)
        for i in range(cols):
            s = exact.storage_to_fraction(sc[r, i // gs], sdt)
            b = exact.storage_to_fraction(bi[r, i // gs], sdt)
            v = _fraction_dequant(codes[i], s, b)
            assert Fraction(float(out32[r, i])) == v
            assert exact.bf16_bits_to_fraction(outbf[r, i]) == exact.rbf16(v)
            assert exact.f16_bits_to_fraction(outh[r, i]) == exact.rf16(v)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("gs", GROUPS)
def test_round_trip_bound_f32_storage(bits, gs):
    """|w - w_hat| <= s/2 (+1 ulp of w_hat), the per-group form of the page's
    round-trip tolerance test."""
    rng = np.random.default_rng(100 + bits + gs)
    rows, cols = 8, 2 * gs
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    packed, sc, bi = oracle.quantize(w, oracle.F32, gs, bits, oracle.F32)
    deq = oracle.dequantize(packed, sc, bi, oracle.F32, cols, gs, bits, oracle.F32)
    s = np.repeat(sc.astype(np.float64), gs, axis=1)
    err = np.abs(deq.astype(np.float64) - w)
    ulp = np.spacing(np.abs(deq)).astype(np.float64)
    assert np.all(err <= s / 2 + ulp)
    # the bias is the group minimum and the codes reach both ends of the range
    mn = w.reshape(rows, -1, gs).min(axis=2)
    assert np.array_equal(bi, mn)
    codes = np.array([exact.unpack_bigint(packed[r].tolist(), bits, cols) for r in range(rows)])
    assert codes.reshape(rows, -1, gs).min(axis=2).max() == 0
    assert codes.reshape(rows, -1, gs).max(axis=2).min() == (1 << bits) - 1


@pytest.mark.parametrize("bits", BITS)
def test_round_trip_bound_bf16_storage(bits):
    gs = 64
    rng = np.random.default_rng(200 + bits)
    rows, cols = 8, 4 * gs
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    packed, sc, bi = oracle.quantize(w, oracle.F32, gs, bits, oracle.BF16)
    deq = oracle.dequantize(packed, sc, bi, oracle.BF16, cols, gs, bits, oracle.F32)
    wg = w.reshape(rows, -1, gs).astype(np.float64)
    mn, mx = wg.min(axis=2), wg.max(axis=2)
    scale_f = ((mx - mn) / ((1 << bits) - 1)).astype(np.float32).astype(np.float64)
    s, b = widen(sc, "bf16"), widen(bi, "bf16")
    bound = s / 2 + np.abs(b - mn) + ((1 << bits) - 1) * np.abs(s - scale_f)
    err = np.abs(deq.astype(np.float64).reshape(rows, -1, gs) - wg).max(axis=2)
    assert np.all(err <= bound * (1 + 1e-6) + 1e-9)


def _exact_grid_distance(wv, q, s, b):
    return abs(wv - (q * s + b))


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("sdt", ["bf16", "f16"])
def test_codes_are_nearest_on_the_stored_grid(bits, sdt):
    """Every code picks the point of its group's STORED grid {q*s + b, 0 <= q < 2^b}
    nearest to w (exact rationals; the slack covers the two fp32 roundings of
    (w - b)/s).  This holds only if codes are computed against the rounded
    scale and bias, and clamped at both ends.  Group 0 of row 0 is built so
    that its fp32 scale 1 + 2^-8 - 2^-20 rounds down to 1 in bf16: its top
    value then sits 2^b/256 codes above the last code, past 255.5 at 8 bits."""
    gs, rows, cols = 64, 16, 128
    qmax = (1 << bits) - 1
    rng = np.random.default_rng(400 + bits)
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    scale_f = np.float32(1.0 + 2.0**-8 - 2.0**-20)
    top = np.float32(np.float64(scale_f) * qmax)
    w[0, :gs] = (rng.random(gs) * float(top)).astype(np.float32)
    w[0, 0], w[0, 1] = 0.0, top
    packed, sc, bi = oracle.quantize(w, oracle.F32, gs, bits, DT[sdt])
    if sdt == "bf16":
        assert widen(sc, sdt)[0, 0] == 1.0
    for r in range(rows):
        codes = exact.unpack_bigint(packed[r].tolist(), bits, cols)
        for i in range(cols):
            s = exact.storage_to_fraction(sc[r, i // gs], sdt)
            b = exact.storage_to_fraction(bi[r, i // gs], sdt)
            wv, q = Fraction(float(w[r, i])), codes[i]
            d = _exact_grid_distance(wv, q, s, b)
            slack = s * (qmax + 1) * Fraction(1, 2**22)
            for qn in (q - 1, q + 1):
                if 0 <= qn <= qmax:
                    assert d <= _exact_grid_distance(wv, qn, s, b) + slack, (r, i, q)
    assert exact.unpack_bigint(packed[0].tolist(), bits, cols)[1] == qmax


def test_tie_rounds_half_away_from_zero():
    """{0, 6.5, 7.5, 15, 0...}: s = 1, so codes are 0, 7, 8, 15 under half-away
    (half-even would give 6 for 6.5)."""
    w = np.zeros((1, 32), dtype=np.float32)
    w[0, 1], w[0, 2], w[0, 3] = 6.5, 7.5, 15.0
    packed, sc, bi = oracle.quantize(w, oracle.F32, 32, 4, oracle.F32)
    assert sc[0, 0] == 1.0 and bi[0, 0] == 0.0
    codes = exact.unpack_bigint(packed[0].tolist(), 4, 32)
    assert codes[:4] == [0, 7, 8, 15]


def test_constant_group_is_exact():
    """A constant group: scale floored at FLT_EPSILON, all codes 0, w_hat = c."""
    for c in (0.0, -0.0, 0.75, -3.0):
        w = np.full((2, 64), c, dtype=np.float32)
        packed, sc, bi = oracle.quantize(w, oracle.F32, 64, 4, oracle.F32)
        assert np.all(sc == np.float32(np.finfo(np.float32).eps))
        assert np.all(packed == 0)
        deq = oracle.dequantize(packed, sc, bi, oracle.F32, 64, 64, 4, oracle.F32)
        assert np.all(deq == np.float32(c))
        if c == 0.0:
            assert not np.any(np.signbit(bi)), "bias -0 must be stored as +0"


def test_rejects_unsupported_params():
    w = np.zeros((1, 96), dtype=np.float32)
    for bits, gs in ((5, 32), (4, 48), (1, 32), (4, 16)):
        with pytest.raises(ValueError):
            oracle.quantize(w, oracle.F32, gs, bits, oracle.F32)


# ------------------------------------------------------------------ the iota example
def _iota_expected():
    """quantized_matmul(iota{3,128}, from_dense(iota{4,128})) computed with exact
    rationals: group min/max, fp32 scale, codes, fp32 fmaf dequant, exact sum."""
    gs, bits = 64, 4
    W = [[Fraction(128 * r + c) for c in range(128)] for r in range(4)]
    X = [[Fraction(128 * r + c) for c in range(128)] for r in range(3)]
    what = []
    for r in range(4):
        row = []
        for g in range(2):
            vals = W[r][g * gs:(g + 1) * gs]
            mn, mx = min(vals), max(vals)
            s = exact.rf32(exact.rf32(mx - mn) / 15)
            b = exact.rf32(mn)
            for v in vals:
                t = exact.rf32(exact.rf32(v - b) / s)
                q = min(max(exact.round_half_away(t), 0), 15)
                row.append(exact.rf32(q * s + b))
        what.append(row)
    y = [[sum(X[m][k] * what[n][k] for k in range(128)) for n in range(4)] for m in range(3)]
    ydense = [[sum(X[m][k] * W[n][k] for k in range(128)) for n in range(4)] for m in range(3)]
    return what, y, ydense


def test_iota_example_quantized_matmul():
    ex = GOLDEN["quantized_matmul_iota"]
    d = ex["from_dense_defaults"]
    w = wl.iota(*ex["w_shape"]).numpy()
    x = wl.iota(*ex["x_shape"]).numpy()
    packed, sc, bi = oracle.quantize(w, oracle.F32, d["group_size"], d["bits"], oracle.F32)
    y = oracle.matmul(x, oracle.F32, packed, sc, bi, oracle.F32, ex["w_shape"][0],
                      d["group_size"], d["bits"])
    assert list(y.shape) == ex["y_shape"]
    what, y_exact, y_dense = _iota_expected()
    deq = oracle.dequantize(packed, sc, bi, oracle.F32, 128, 64, 4, oracle.F32)
    assert [[Fraction(float(v)) for v in row] for row in deq] == what
    for m in range(3):
        for n in range(4):
            bound = 128 * 2.0**-53 * float(sum(abs(x[m, k]) * abs(deq[n, k]) for k in range(128)))
            assert abs(Fraction(y[m, n]) - y_exact[m][n]) <= Fraction(bound)
            # quantized result stays within the round-trip bound of the dense product
            assert abs(y[m, n] - float(y_dense[m][n])) <= float(np.abs(x[m]).sum()) * 4.2 / 2
    # first entry, hand-checkable: scale = fp32(63/15), dense x0.w0 = 690880
    assert float(sc[0, 0]) == float(np.float32(4.2))
    assert float(y_dense[0][0]) == 690880.0


def test_iota_example_dequantize_shape():
    ex = GOLDEN["dequantize_defn_iota"]
    w = wl.iota(*ex["w_shape"]).numpy()
    packed, sc, bi = oracle.quantize(w, oracle.F32, ex["group_size"], ex["bits"], oracle.F32)
    deq = oracle.dequantize(packed, sc, bi, oracle.F32, w.shape[1], ex["group_size"], ex["bits"],
                            oracle.F32)
    assert list(deq.shape) == ex["dense_shape"]
    assert np.abs(deq - w).max() <= 4.2 / 2


# ------------------------------------------------------------------ matmul brute force
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("transpose", [True, False])
def test_matmul_brute_force_exact(bits, transpose):
    rng = np.random.default_rng(300 + bits + int(transpose))
    gs = 32
    M, N, K = 3, 5 if transpose else 64, 64 if transpose else 7
    qrows, qcols = (N, K) if transpose else (K, N)
    w = (rng.standard_normal((qrows, qcols)) * 0.02).astype(np.float32)
    x = wl.storage_numpy(torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16))
    packed, sc, bi = oracle.quantize(w, oracle.F32, gs, bits, oracle.BF16)
    y = oracle.matmul(x, oracle.BF16, packed, sc, bi, oracle.BF16, N, gs, bits, transpose)
    deq = oracle.dequantize(packed, sc, bi, oracle.BF16, qcols, gs, bits, oracle.F32)
    wd = deq if transpose else deq.T  # wd[n][k]
    xf = widen(x, "bf16")
    for m in range(M):
        for n in range(N):
            terms = [Fraction(xf[m, k]) * Fraction(float(wd[n, k])) for k in range(K)]
            ex_sum = sum(terms)
            bound = K * 2.0**-53 * float(sum(abs(t) for t in terms))
            assert abs(Fraction(y[m, n]) - ex_sum) <= Fraction(bound)
    coords = [(0, 0), (M - 1, N - 1), (1, 2)]
    el = oracle.matmul_elements(x, oracle.BF16, packed, sc, bi, oracle.BF16, N, gs, bits, coords,
                                transpose)
    assert np.array_equal(el, np.array([y[m, n] for m, n in coords]))


def test_matmul_orientations_agree():
    """Both layouts against numpy fp64 products of the oracle's own dequantized
    matrices: transpose=1 is x . W^T with W [N, K]; transpose=0 is x . W with
    W [K, N] quantized along N."""
    rng = np.random.default_rng(9)
    gs, bits = 32, 4
    w = (rng.standard_normal((32, 32)) * 0.02).astype(np.float32)
    x = rng.standard_normal((2, 32)).astype(np.float32)
    p1, s1, b1 = oracle.quantize(w, oracle.F32, gs, bits, oracle.F32)
    d1 = oracle.dequantize(p1, s1, b1, oracle.F32, 32, gs, bits, oracle.F32)
    y1 = oracle.matmul(x, oracle.F32, p1, s1, b1, oracle.F32, 32, gs, bits, True)
    assert np.allclose(y1, x.astype(np.float64) @ d1.astype(np.float64).T, rtol=1e-12, atol=1e-12)
    p0, s0, b0 = oracle.quantize(np.ascontiguousarray(w.T), oracle.F32, gs, bits, oracle.F32)
    d0 = oracle.dequantize(p0, s0, b0, oracle.F32, 32, gs, bits, oracle.F32)  # [K, N]
    y0 = oracle.matmul(x, oracle.F32, p0, s0, b0, oracle.F32, 32, gs, bits, False)
    assert np.allclose(y0, x.astype(np.float64) @ d0.astype(np.float64), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ MoE
def _stack(E, n_rows, n_cols, bits, gs, seed, sdt="bf16"):
    w = wl.gen_weight(E * n_rows, n_cols, seed).numpy()
    packed, sc, bi = oracle.quantize(w, oracle.F32, gs, bits, DT[sdt])
    st = oracle.Stack(packed, sc, bi, DT[sdt], E, n_rows, n_cols, gs, bits)
    deq = oracle.dequantize(packed, sc, bi, DT[sdt], n_cols, gs, bits, oracle.F32)
    return st, deq.astype(np.float64).reshape(E, n_rows, n_cols)


def test_moe_gemv_id_equals_per_pair_loop():
    E, n_rows, n_cols, bits, gs = 6, 16, 64, 4, 32
    st, deq = _stack(E, n_rows, n_cols, bits, gs, 11)
    n_sel, stride = 5, 64
    a = wl.storage_numpy(wl.gen_x(n_sel, n_cols, 12))
    ids = np.array([3, 0, 5, 3, 1], dtype=np.int32)
    out, rc = oracle.moe_gemv_id(a.reshape(-1), oracle.BF16, ids, n_sel, stride, st)
    assert rc == oracle.ORC_OK
    af = widen(a.reshape(-1), "bf16")
    for i in range(n_sel):
        ref = deq[ids[i]] @ af[i * stride:i * stride + n_cols]
        assert np.allclose(out[i], ref, rtol=1e-12, atol=1e-14)


def test_moe_batched_offsets_follow_the_page_formula():
    E, n_rows, n_cols, bits, gs = 5, 8, 64, 3, 32
    st, deq = _stack(E, n_rows, n_cols, bits, gs, 21)
    m, top_k, outer, inner = 3, 2, 200, 70
    a = wl.storage_numpy(wl.gen_x(1, outer * m + 10, 22)).reshape(-1)
    ids = np.array([[1, 4], [0, 0], [2, 3]], dtype=np.int32)
    out, rc = oracle.moe_gemv_id_batched(a, oracle.BF16, ids, m, top_k, outer, inner, st)
    assert rc == oracle.ORC_OK
    af = widen(a, "bf16")
    for p in range(m * top_k):
        off = (p // top_k) * outer + (p % top_k) * inner
        ref = deq[ids.reshape(-1)[p]] @ af[off:off + n_cols]
        assert np.allclose(out[p], ref, rtol=1e-12, atol=1e-14)


def test_moe_all_same_expert_equals_matmul():
    E, n_rows, n_cols, bits, gs = 4, 16, 128, 4, 64
    st, deq = _stack(E, n_rows, n_cols, bits, gs, 31)
    e = 2
    a = wl.storage_numpy(wl.gen_x(3, n_cols, 32))
    out, rc = oracle.moe_gemv_id(a.reshape(-1), oracle.BF16, np.full(3, e, np.int32), 3, n_cols, st)
    G = n_cols // gs
    y = oracle.matmul(a, oracle.BF16, st.packed[e * n_rows:(e + 1) * n_rows],
                      np.ascontiguousarray(st.scales[e * n_rows:(e + 1) * n_rows]),
                      np.ascontiguousarray(st.biases[e * n_rows:(e + 1) * n_rows]), oracle.BF16,
                      n_rows, gs, bits)
    assert G == 2 and rc == oracle.ORC_OK
    assert np.array_equal(out, y)


def test_moe_gate_up_silu_closed_form():
    E, n_rows, n_cols, bits, gs = 4, 8, 64, 4, 32
    gate, dg = _stack(E, n_rows, n_cols, bits, gs, 41)
    up, du = _stack(E, n_rows, n_cols, bits, gs, 42)
    a = wl.storage_numpy(wl.gen_x(1, n_cols, 43)).reshape(-1)
    ids = np.array([1, 3, 1], dtype=np.int32)
    out, rc = oracle.moe_gate_up_silu(a, oracle.BF16, ids, 3, gate, up)
    assert rc == oracle.ORC_OK
    af = widen(a, "bf16")
    for i, e in enumerate(ids):
        g, u = dg[e] @ af, du[e] @ af
        ref = g / (1.0 + np.exp(-g)) * u
        assert np.allclose(out[i], ref, rtol=1e-12, atol=1e-15)
    # SiLU(0) * u = 0: zero activations give exactly zero
    z = np.zeros_like(a)
    out0, _ = oracle.moe_gate_up_silu(z, oracle.BF16, ids, 3, gate, up)
    assert np.all(out0 == 0.0)
    # batched form with pair offsets
    m, top_k, outer, inner = 2, 2, 64, 0
    a2 = wl.storage_numpy(wl.gen_x(2, n_cols, 44)).reshape(-1)
    ids2 = np.array([[0, 2], [3, 3]], dtype=np.int32)
    ob, rc = oracle.moe_gate_up_silu_batched(a2, oracle.BF16, ids2, m, top_k, outer, inner, gate, up)
    af2 = widen(a2, "bf16")
    for p in range(4):
        e = ids2.reshape(-1)[p]
        off = (p // top_k) * outer + (p % top_k) * inner
        g, u = dg[e] @ af2[off:off + n_cols], du[e] @ af2[off:off + n_cols]
        assert np.allclose(ob[p], g / (1 + np.exp(-g)) * u, rtol=1e-12, atol=1e-15)


def test_moe_bad_id_reports_and_zero_fills():
    E, n_rows, n_cols, bits, gs = 3, 8, 64, 4, 32
    st, _ = _stack(E, n_rows, n_cols, bits, gs, 51)
    a = wl.storage_numpy(wl.gen_x(1, n_cols, 52)).reshape(-1)
    out, rc = oracle.moe_gemv_id(a, oracle.BF16, np.array([0, 7, -1], np.int32), 3, 0, st)
    assert rc == oracle.ORC_ERR_ID
    assert np.all(out[1] == 0) and np.all(out[2] == 0) and np.any(out[0] != 0)
    # the same rule in the batched and fused forms
    ids2 = np.array([[0, 3], [-2, 1]], np.int32)
    ob, rc = oracle.moe_gemv_id_batched(a, oracle.BF16, ids2, 2, 2, 0, 0, st)
    assert rc == oracle.ORC_ERR_ID
    assert np.all(ob[1] == 0) and np.all(ob[2] == 0) and np.any(ob[0] != 0) and np.any(ob[3] != 0)
    og, rc = oracle.moe_gate_up_silu(a, oracle.BF16, np.array([3, 2], np.int32), 2, st, st)
    assert rc == oracle.ORC_ERR_ID
    assert np.all(og[0] == 0) and np.any(og[1] != 0)
    ogb, rc = oracle.moe_gate_up_silu_batched(a, oracle.BF16, ids2, 2, 2, 0, 0, st, st)
    assert rc == oracle.ORC_ERR_ID
    assert np.all(ogb[1] == 0) and np.all(ogb[2] == 0) and np.any(ogb[0] != 0)


@pytest.mark.parametrize("x_dtype", [oracle.BF16, oracle.F16, oracle.F32])
def test_widen_f64_matches_the_scalar_conversions(x_dtype):
    """the vector widening used by matmul_dense equals the C conversions"""
    rng = np.random.default_rng(7)
    if x_dtype == oracle.F32:
        x = rng.standard_normal(64).astype(np.float32)
        ref = x.astype(np.float64)
    else:
        x = rng.integers(0, 1 << 16, 256, dtype=np.uint16)
        x = x[(x & 0x7C00) != 0x7C00] if x_dtype == oracle.F16 else x[(x & 0x7F80) != 0x7F80]
        conv = oracle.bf16_to_f32 if x_dtype == oracle.BF16 else oracle.f16_to_f32
        ref = np.array([conv(int(h)) for h in x], dtype=np.float64)
    assert np.array_equal(oracle.widen_f64(x, x_dtype), ref)


@pytest.mark.parametrize("bits", [3, 4, 8])
def test_matmul_dense_agrees_with_matmul(bits):
    """the library-GEMM form and the plain loops compute the same sums: they
    differ only by summation order, within K * 2^-53 * sum |x| |w|"""
    N, K, M, gs = 48, 256, 7, 64
    w = wl.gen_weight(N, K, 30 + bits).numpy()
    p, s, b = oracle.quantize(w, oracle.F32, gs, bits, oracle.BF16)
    x = wl.storage_numpy(wl.gen_x(M, K, 31))
    y1 = oracle.matmul(x, oracle.BF16, p, s, b, oracle.BF16, N, gs, bits)
    y2 = oracle.matmul_dense(x, oracle.BF16, p, s, b, oracle.BF16, N, gs, bits)
    wd = oracle.dequantize(p, s, b, oracle.BF16, K, gs, bits, oracle.F32).astype(np.float64)
    bound = K * 2.0 ** -52 * (np.abs(oracle.widen_f64(x, oracle.BF16)) @ np.abs(wd).T)
    assert np.all(np.abs(y1 - y2) <= bound)
    # a dropped term would show: zeroing one weight column changes y2 beyond the bound
    p2 = p.copy()
    p2[:, 0] = 0
    y3 = oracle.matmul_dense(x, oracle.BF16, p2, s, b, oracle.BF16, N, gs, bits)
    assert np.any(np.abs(y3 - y1) > bound)


@pytest.mark.parametrize("outer_inner", [(64, 0), (4 * 64, 64)])
def test_moe_batched_dense_agrees_with_the_loops(outer_inner):
    """the per-expert library-GEMM form of the MoE oracle equals the plain
    per-pair loops within fp64 summation-order error; bad ids zero-filled"""
    E, n_rows, n_cols, bits, gs, m, top_k = 6, 24, 64, 4, 32, 5, 4
    outer, inner = outer_inner
    w = wl.gen_weight(E * n_rows, n_cols, 41).numpy()
    p, s, b = oracle.quantize(w, oracle.F32, gs, bits, oracle.BF16)
    st = oracle.Stack(p, s, b, oracle.BF16, E, n_rows, n_cols, gs, bits)
    a = wl.storage_numpy(wl.gen_x(1, m * outer + top_k * inner + n_cols, 42)).reshape(-1)
    ids = wl.gen_moe_ids(m, E, top_k, 43).numpy()
    ids[2, 1] = E + 3  # an out-of-range id
    ref, rc = oracle.moe_gemv_id_batched(a, oracle.BF16, ids, m, top_k, outer, inner, st)
    got, rc2 = oracle.moe_batched_dense(a, oracle.BF16, ids, m, top_k, outer, inner, st)
    assert rc == rc2 == oracle.ORC_ERR_ID
    assert np.all(got[2 * top_k + 1] == 0)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)
    # a swapped offset (inner and outer exchanged) is caught
    if inner:
        bad, _ = oracle.moe_batched_dense(a, oracle.BF16, ids, m, top_k, inner, outer, st)
        assert not np.allclose(bad, ref, rtol=0, atol=1e-6)


# ------------------------------------------------------------------ microscaled modes
def test_fp4_e2m1_matches_the_printed_table():
    tab = GOLDEN["fp4_e2m1_table"]["value"]
    got = [oracle.fp4_e2m1(c) for c in range(16)]
    assert got == tab
    assert [math.copysign(1.0, v) for v in got] == [math.copysign(1.0, v) for v in tab]  # -0.0 kept


def test_e8m0_is_two_to_the_byte_minus_127():
    bias = GOLDEN["e8m0_rule"]["bias"]
    for s in range(256):
        exp = math.ldexp(1.0, s - bias)
        got = oracle.e8m0(s)
        assert (got == exp) if exp < 3.4e38 else math.isinf(got)


def test_fp8_e4m3_matches_the_format_and_the_page():
    """every finite OCP E4M3 byte decodes as torch's float8_e4m3fn does; the
    two bytes that format calls NaN decode to +-480 as the page states"""
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float32).tolist()
    sat = GOLDEN["fp8_e4m3_saturation"]
    for i in range(256):
        got = oracle.fp8_e4m3(i)
        if i in (0x7F, 0xFF):
            assert got == sat[f"0x{i:02x}"]
        else:
            assert got == ref[i] and math.copysign(1.0, got) == math.copysign(1.0, ref[i])


@pytest.mark.parametrize("mode", [oracle.MODE_MXFP4, oracle.MODE_MXFP8, oracle.MODE_NVFP4])
def test_dequant_mx_exact_rational(mode):
    """w_hat = lane(q) * scale(s) exactly (the products are exact in fp32),
    lanes read LSB-first, one scale per group of the mode's group size"""
    preset = GOLDEN["microscaled_presets"][{1: "mxfp4", 2: "mxfp8", 3: "nvfp4"}[mode]]
    bits, gs = oracle.MX_PARAMS[mode]
    assert (bits, gs) == (preset["bits"], preset["group_size"])
    rows, cols = 5, 4 * gs
    rng = np.random.default_rng(11 + mode)
    codes = rng.integers(0, 1 << bits, (rows, cols), dtype=np.uint8)
    if mode == oracle.MODE_MXFP8:
        codes[codes == 0x7F] = 0x7E  # keep the saturation bytes out of the exactness check
    if mode == oracle.MODE_NVFP4:
        sc = rng.integers(0, 0x7E, (rows, cols // gs), dtype=np.uint8)  # positive E4M3 scales
    else:
        sc = rng.integers(100, 150, (rows, cols // gs), dtype=np.uint8)
    packed = np.stack([oracle.pack_row(r, bits) for r in codes])
    out = oracle.dequantize_mx(packed, sc, mode, cols, oracle.F32)
    lane = (lambda c: oracle.fp8_e4m3(c)) if mode == oracle.MODE_MXFP8 else (lambda c: oracle.fp4_e2m1(c))
    scl = (lambda s: oracle.fp8_e4m3(s)) if mode == oracle.MODE_NVFP4 else (lambda s: oracle.e8m0(s))
    for r in range(rows):
        for i in range(cols):
            exp = Fraction(lane(int(codes[r, i]))) * Fraction(scl(int(sc[r, i // gs])))
            assert Fraction(float(out[r, i])) == exp


@pytest.mark.parametrize("mode", [oracle.MODE_MXFP4, oracle.MODE_MXFP8, oracle.MODE_NVFP4])
def test_matmul_mx_brute_force(mode):
    bits, gs = oracle.MX_PARAMS[mode]
    N, K, M = 6, 2 * gs, 3
    rng = np.random.default_rng(21 + mode)
    codes = rng.integers(0, 1 << bits, (N, K), dtype=np.uint8)
    sc = rng.integers(110, 130, (N, K // gs), dtype=np.uint8) if mode != oracle.MODE_NVFP4 else \
        rng.integers(0x20, 0x50, (N, K // gs), dtype=np.uint8)
    packed = np.stack([oracle.pack_row(r, bits) for r in codes])
    x = wl.storage_numpy(wl.gen_x(M, K, 22))
    y = oracle.matmul_mx(x, oracle.BF16, packed, sc, mode, N)
    wd = oracle.dequantize_mx(packed, sc, mode, K, oracle.F32).astype(np.float64)
    xs = oracle.widen_f64(x, oracle.BF16)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xs[m, k])) * Fraction(float(wd[n, k])) for k in range(K))
            bound = K * 2.0 ** -52 * float(np.abs(xs[m]) @ np.abs(wd[n]))
            assert abs(float(exact) - y[m, n]) <= bound


# ------------------------------------------------------------------ per-tensor dynamic int8
def test_dynamic_int8_page_round_trip():
    """the page's own fixture: every element comes back within one step + 1e-4"""
    g = GOLDEN["dynamic_int8_round_trip"]
    w = np.array(g["weights"], dtype=np.float32)
    q, params = oracle.quantize_dynamic_int8(w, oracle.F32)
    assert params.tolist() == [w.min(), w.max(), w.min(), w.max()]
    back = oracle.dequantize_dynamic_int8(q, params, oracle.F32)
    tol = (params[3] - params[2]) / g["divisor"] + g["extra_tol"]
    assert np.all(np.abs(back.astype(np.float64) - w) <= tol)
    lo, hi = g["code_range"]
    assert q.min() == lo and q.max() == hi  # the extremes land on the end codes


def test_dynamic_int8_dequant_exact_rational():
    """w_hat = fl(fl(fl(q + 128) * scale) + min), scale = fl((max - min) / 255):
    each fp32 operation rounded once, checked with exact rationals"""
    rng = np.random.default_rng(5)
    q = rng.integers(-128, 128, 300, dtype=np.int8)
    for mn, mx in [(-0.37, 0.81), (-3.0, -1.0), (1e-3, 2e-3), (-1e4, 3e4)]:
        params = np.array([mn, mx, mn, mx], dtype=np.float32)
        out = oracle.dequantize_dynamic_int8(q, params, oracle.F32)
        f32 = lambda fr: Fraction(float(np.float32(float(fr))))  # noqa: E731  round to nearest fp32
        scale = f32(Fraction(float(params[3])) - Fraction(float(params[2])))
        scale = f32(scale / 255)
        for i in range(q.size):
            sh = Fraction(int(q[i]) + 128)
            exp = f32(f32(sh * scale) + Fraction(float(params[2])))
            assert Fraction(float(out[i])) == exp


def test_dynamic_int8_codes_are_nearest():
    """each code is the nearest point of the affine 256-point grid (brute force
    over all 256 codes, ties allowed either way within the fp32 rounding)"""
    rng = np.random.default_rng(6)
    w = (rng.standard_normal(513) * 0.7).astype(np.float32)
    q, params = oracle.quantize_dynamic_int8(w, oracle.F32)
    mn = float(params[0])
    scale = float(np.float32((np.float32(params[1]) - np.float32(params[0])) / np.float32(255)))
    grid = np.arange(256, dtype=np.float64) * scale + mn
    for i in range(w.size):
        d = np.abs(grid - float(w[i]))
        best = d.min()
        assert d[int(q[i]) + 128] <= best + 1e-6 * scale


def test_dynamic_int8_constant_tensor():
    """max == min: the scale floor FLT_EPSILON keeps it finite; all codes -128
    and the dequantized tensor is the constant exactly"""
    w = np.full(40, 0.625, dtype=np.float32)
    q, params = oracle.quantize_dynamic_int8(w, oracle.F32)
    assert np.all(q == -128)
    back = oracle.dequantize_dynamic_int8(q, params, oracle.F32)
    assert np.all(back == np.float32(0.625))


def test_dynamic_int8_matmul_brute_force():
    rng = np.random.default_rng(7)
    N, K, M = 5, 96, 3
    w = (rng.standard_normal((N, K)) * 0.3).astype(np.float32)
    q, params = oracle.quantize_dynamic_int8(w, oracle.F32)
    x = wl.storage_numpy(wl.gen_x(M, K, 8))
    y = oracle.matmul_dynamic_int8(x, oracle.BF16, q, params)
    wd = oracle.dequantize_dynamic_int8(q, params, oracle.F32).astype(np.float64)
    xs = oracle.widen_f64(x, oracle.BF16)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xs[m, k])) * Fraction(float(wd[n, k])) for k in range(K))
            bound = K * 2.0 ** -52 * float(np.abs(xs[m]) @ np.abs(wd[n]))
            assert abs(float(exact) - y[m, n]) <= bound


def test_dynamic_int8_nan_elements_follow_the_page_fold():
    """NaN elements take no part in min/max (f32::min / f32::max skip NaN) and
    quantize to code 0 (a NaN float cast to i8 is 0); the other codes are the
    ones the tensor without them gets"""
    w = np.array([0.5, np.nan, -1.0, 2.0, np.nan, 0.0], dtype=np.float32)
    q, params = oracle.quantize_dynamic_int8(w, oracle.F32)
    assert params.tolist() == [-1.0, 2.0, -1.0, 2.0]
    assert q[1] == 0 and q[4] == 0
    q2, _ = oracle.quantize_dynamic_int8(w[~np.isnan(w)], oracle.F32)
    assert q[~np.isnan(w)].tolist() == q2.tolist()
