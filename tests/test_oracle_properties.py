"""Property tests of the oracle quantizer over generated weights (no GPU).

Hypothesis draws the shape parameters, a value distribution per group
(normal at a random magnitude, all-negative, heavy-tailed, near-constant)
and the input and storage dtypes.  For every draw the oracle must satisfy
what the per-group min/max rule fixes whatever the values:
  - the bias is the group minimum rounded once to the storage dtype;
  - the scale is max((max - min)/(2^b - 1), FLT_EPSILON) rounded once;
  - every code is the nearest point of the stored grid {q*s + b};
  - bf16 or f16 weights quantize exactly as their (exact) f32 widening.
Exact rationals decide each comparison.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from tests import exact
from weight_only_quantized_qmm_b200 import workloads as wl

DT = {"f32": oracle.F32, "f16": oracle.F16, "bf16": oracle.BF16}
TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
FLT_EPS = Fraction(2) ** -23


def _storage_fraction(arr, i, sdt):
    return exact.storage_to_fraction(arr.reshape(-1)[i], sdt)


def _round_to(v: Fraction, sdt: str) -> Fraction:
    return {"f32": exact.rf32, "bf16": exact.rbf16, "f16": exact.rf16}[sdt](v)


@st.composite
def weights(draw):
    bits = draw(st.sampled_from([2, 3, 4, 6, 8]))
    gs = draw(st.sampled_from([32, 64, 128]))
    groups = draw(st.integers(1, 3))
    rows = draw(st.integers(1, 3))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    cols = groups * gs
    w = np.empty((rows, cols), dtype=np.float64)
    for r in range(rows):
        for g in range(groups):
            kind = draw(st.sampled_from(["normal", "negative", "heavy", "flat"]))
            mag = 10.0 ** draw(st.integers(-4, 3))
            if kind == "normal":
                v = rng.standard_normal(gs) * mag
            elif kind == "negative":
                v = -np.abs(rng.standard_normal(gs)) * mag - mag
            elif kind == "heavy":
                v = rng.standard_cauchy(gs) * mag
            else:
                v = mag + rng.standard_normal(gs) * mag * 1e-6
            w[r, g * gs:(g + 1) * gs] = v
    wdt = draw(st.sampled_from(["f32", "bf16", "f16"]))
    sdt = draw(st.sampled_from(["f32", "bf16", "f16"]))
    if wdt == "f16" or sdt == "f16":
        w = np.clip(w, -60000.0, 60000.0)  # keep groups finite in binary16
    return bits, gs, wdt, sdt, torch.from_numpy(w).to(TORCH_DT[wdt])


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(weights())
def test_quantizer_properties(case):
    bits, gs, wdt, sdt, wt = case
    rows, cols = wt.shape
    qmax = (1 << bits) - 1
    w_store = wl.storage_numpy(wt)
    packed, sc, bi = oracle.quantize(w_store, DT[wdt], gs, bits, DT[sdt])
    # the same values given as f32 (an exact widening) quantize identically
    w32 = wt.to(torch.float32).numpy()
    p32, s32, b32 = oracle.quantize(w32, oracle.F32, gs, bits, DT[sdt])
    assert np.array_equal(packed, p32) and np.array_equal(sc, s32) and np.array_equal(bi, b32)
    G = cols // gs
    for r in range(rows):
        codes = exact.unpack_bigint(packed[r].tolist(), bits, cols)
        for g in range(G):
            vals = [Fraction(float(v)) for v in w32[r, g * gs:(g + 1) * gs]]
            mn, mx = min(vals), max(vals)
            s = _storage_fraction(sc, r * G + g, sdt)
            b = _storage_fraction(bi, r * G + g, sdt)
            assert b == _round_to(mn, sdt)
            scale_f = max(exact.rf32(exact.rf32(mx - mn) / qmax), FLT_EPS)
            assert s == _round_to(scale_f, sdt)
            slack = s * (qmax + 1) * Fraction(1, 2**22)
            for i, wv in enumerate(vals):
                q = codes[g * gs + i]
                assert 0 <= q <= qmax
                d = abs(wv - (q * s + b))
                for qn in (q - 1, q + 1):
                    if 0 <= qn <= qmax:
                        assert d <= abs(wv - (qn * s + b)) + slack, (r, g, i, q)
