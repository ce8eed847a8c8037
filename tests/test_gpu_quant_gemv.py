"""GPU parity: quantize, dequantize and the decode-shaped matmul against the
CPU oracle, through the C ABI (libqmm.so via the ctypes binding)."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import ORC, Guarded, gate, np_storage, packed_np, qweight_np, rne_equal
from weight_only_quantized_qmm_b200 import api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
BITS = [2, 3, 4, 6, 8]
GROUPS = [32, 64, 128]
DEV = "cuda"


def _quant_pair(n, k, bits, gs, s_dtype, seed, w_dtype=torch.float32):
    w = wl.gen_weight(n, k, seed).to(w_dtype)
    qw = api.qmm_quantize(w.to(DEV), gs, bits, s_dtype)
    torch.cuda.synchronize()
    ref = oracle.quantize(np_storage(w), ORC[w_dtype], gs, bits, ORC[s_dtype])
    return w, qw, ref


# ------------------------------------------------------------------ quantize / dequantize
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("gs", GROUPS)
@pytest.mark.parametrize("s_dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_quantize_bit_exact(bits, gs, s_dtype):
    _, qw, (p_ref, s_ref, b_ref) = _quant_pair(37, 4 * gs, bits, gs, s_dtype, 10 + bits + gs)
    p, s, b = qweight_np(qw)
    assert np.array_equal(p, p_ref), "packed words differ"
    assert np.array_equal(s, s_ref), "scales differ"
    assert np.array_equal(b, b_ref), "biases differ"


@pytest.mark.parametrize("w_dtype", [torch.bfloat16, torch.float16])
def test_quantize_half_inputs_bit_exact(w_dtype):
    _, qw, (p_ref, s_ref, b_ref) = _quant_pair(64, 256, 4, 64, w_dtype, 5, w_dtype)
    p, s, b = qweight_np(qw)
    assert np.array_equal(p, p_ref) and np.array_equal(s, s_ref) and np.array_equal(b, b_ref)


def test_quantize_degenerate_groups():
    """constant groups, -0.0, on-grid values and a tie of the rounding rule"""
    w = torch.zeros(4, 64)
    w[1] = 0.75
    w[2] = -0.0
    w[3, :4] = torch.tensor([0.0, 6.5, 7.5, 15.0])
    qw = api.qmm_quantize(w.to(DEV), 32, 4, torch.float32)
    torch.cuda.synchronize()
    ref = oracle.quantize(w.numpy(), oracle.F32, 32, 4, oracle.F32)
    for got, exp in zip(qweight_np(qw), ref):
        assert np.array_equal(got, exp)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("gs", GROUPS)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_dequantize_bit_exact(bits, gs, out_dtype):
    _, qw, (p_ref, s_ref, b_ref) = _quant_pair(19, 2 * gs, bits, gs, torch.bfloat16, 40 + bits)
    g = Guarded((19, 2 * gs), out_dtype)
    api.qmm_dequantize(qw, out=g.out)
    torch.cuda.synchronize()
    out = g.check("dequant")
    ref = oracle.dequantize(p_ref, s_ref, b_ref, oracle.BF16, 2 * gs, gs, bits, ORC[out_dtype])
    assert np.array_equal(np_storage(out), ref)


# ------------------------------------------------------------------ decode GEMV (M <= 16)
def _gemv_case(M, N, K, bits, gs, dtype, seed):
    """fp32 and 16-bit outputs of one call each, in poisoned buffers with guard
    bands (every output written, nothing past the end touched)."""
    w, qw, (p, s, b) = _quant_pair(N, K, bits, gs, dtype, seed)
    x = wl.gen_x(M, K, seed + 1, {torch.bfloat16: "bf16", torch.float16: "f16",
                                  torch.float32: "f32"}[dtype])
    g32, g16 = Guarded((M, N), torch.float32), Guarded((M, N), dtype)
    api.qmm_matmul(x.to(DEV), qw, True, out=g32.out)
    api.qmm_matmul(x.to(DEV), qw, True, out=g16.out)
    torch.cuda.synchronize()
    y32, y16 = g32.check("y32"), g16.check("y16")
    yref = oracle.matmul(np_storage(x), ORC[dtype], p, s, b, ORC[dtype], N, gs, bits)
    return y32, y16, yref


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("gs", GROUPS)
def test_gemv_all_widths_and_groups(bits, gs):
    y32, y16, yref = _gemv_case(3, 200, 4 * gs + 2 * gs, bits, gs, torch.bfloat16, 100 + bits + gs)
    gate(y32.cpu().numpy(), yref, f"b{bits} g{gs}")
    rne_equal(y16, y32)


@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 13, 16])
def test_gemv_token_counts(M):
    y32, y16, yref = _gemv_case(M, 333, 1024, 4, 64, torch.bfloat16, 200 + M)
    gate(y32.cpu().numpy(), yref, f"M={M}")
    rne_equal(y16, y32)


@pytest.mark.parametrize("bits", [4, 8, 3])
def test_gemv_fp16(bits):
    y32, y16, yref = _gemv_case(4, 160, 512, bits, 64, torch.float16, 300 + bits)
    gate(y32.cpu().numpy(), yref, "f16")
    rne_equal(y16, y32)


@pytest.mark.parametrize("N,K", [(1, 64), (15, 32), (17, 128), (3000, 64)])
def test_gemv_ragged_shapes(N, K):
    gs = 32 if K % 64 else 64
    y32, y16, yref = _gemv_case(2, N, K, 4, gs, torch.bfloat16, 400 + N)
    gate(y32.cpu().numpy(), yref, f"N={N} K={K}")
    rne_equal(y16, y32)


# Rows the streaming kernel takes (2/4/8-bit whole-word lanes, rows of whole
# 128-byte slices, K/gs a multiple of 8 and at least one unit): every mode
# (one token, up to 8, up to 16), unit widths 16/32/64 groups, the two-nibble
# 8-bit bf16 form, a ragged last row tile (N = 200) and a partly filled last
# unit (K = 2560 at g64: 40 groups = 32 + 8).
@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("gs", GROUPS)
@pytest.mark.parametrize("M", [1, 3, 12])
def test_gemv_streaming_kernel_shapes(bits, gs, M):
    y32, y16, yref = _gemv_case(M, 200, 4096, bits, gs, torch.bfloat16, 600 + 10 * bits + gs + M)
    gate(y32.cpu().numpy(), yref, f"stream b{bits} g{gs} M{M}")
    rne_equal(y16, y32)


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("bits", [4, 8])
def test_gemv_streaming_partial_unit_fp16(M, bits):
    y32, y16, yref = _gemv_case(M, 333, 2560, bits, 64, torch.float16, 700 + M + bits)
    gate(y32.cpu().numpy(), yref, f"stream f16 b{bits} M{M} K=2560")
    rne_equal(y16, y32)


@pytest.mark.parametrize("K", [768, 1280])
@pytest.mark.parametrize("M", [1, 6, 16])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_gemv_streaming_short_rows_cp_async_scales(K, M, dtype):
    """K/gs = 12 or 20 groups (even, not a multiple of 8): the scale and bias
    rows are not 16-byte strided, so they stream by 4-byte copies into 16-group
    units, the last one partly filled."""
    y32, y16, yref = _gemv_case(M, 150, K, 4, 64, dtype, 900 + K + M)
    gate(y32.cpu().numpy(), yref, f"stream K={K} M{M}")
    rne_equal(y16, y32)


def test_gemv_streaming_deterministic():
    """Identical calls give identical bits (fixed reduction order)."""
    w, qw, _ = _quant_pair(14336 // 8, 4096, 4, 64, torch.bfloat16, 800)
    x = wl.gen_x(1, 4096, 801).to(DEV)
    ys = [api.qmm_matmul(x, qw, True, torch.float32) for _ in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


def test_gemv_long_k_chunks_x_staging():
    """M=16 with K large enough that staged x is split into several K chunks."""
    y32, y16, yref = _gemv_case(16, 64, 8192, 8, 32, torch.bfloat16, 500)
    gate(y32.cpu().numpy(), yref, "chunked K")
    rne_equal(y16, y32)


def test_tiny_config():
    """W fp32 [256, 512] ~ N(0, 0.02), g64 b4; x bf16 [4, 512] ~ N(0, 1); seed 0."""
    c = wl.WORKLOADS.tiny
    w = wl.gen_weight(c.N, c.K, c.seed)
    x = wl.gen_x(c.M, c.K, c.seed + 1)
    qw = api.qmm_quantize(w.to(DEV), c.group_size, c.bits, torch.bfloat16)
    y32 = api.qmm_matmul(x.to(DEV), qw, True, torch.float32)
    y16 = api.qmm_matmul(x.to(DEV), qw, True)
    torch.cuda.synchronize()
    p, s, b = oracle.quantize(w.numpy(), oracle.F32, c.group_size, c.bits, oracle.BF16)
    assert np.array_equal(packed_np(qw.packed), p)
    yref = oracle.matmul(np_storage(x), oracle.BF16, p, s, b, oracle.BF16, c.N, c.group_size, c.bits)
    assert tuple(y16.shape) == (4, 256)
    gate(y32.cpu().numpy(), yref, "tiny")
    rne_equal(y16, y32)


def test_iota_example_on_gpu():
    """the page's iota example in fp32 (x and scales f32) -> shape (3, 4)"""
    w = wl.iota(4, 128)
    x = wl.iota(3, 128)
    qw = api.qmm_quantize(w.to(DEV), 64, 4, torch.float32)
    y = api.qmm_matmul(x.to(DEV), qw)
    torch.cuda.synchronize()
    p, s, b = oracle.quantize(w.numpy(), oracle.F32, 64, 4, oracle.F32)
    yref = oracle.matmul(x.numpy(), oracle.F32, p, s, b, oracle.F32, 4, 64, 4)
    assert tuple(y.shape) == (3, 4)
    np.testing.assert_allclose(y.cpu().numpy(), yref, rtol=1e-6)


# ------------------------------------------------------------------ generic paths
@pytest.mark.parametrize("bits", [3, 4, 8])
def test_fp32_activations_and_wide_m(bits):
    M, N, K, gs = 21, 96, 256, 32
    w, qw, (p, s, b) = _quant_pair(N, K, bits, gs, torch.float32, 600 + bits)
    x = wl.gen_x(M, K, 601, "f32")
    y = api.qmm_matmul(x.to(DEV), qw)
    torch.cuda.synchronize()
    yref = oracle.matmul(x.numpy(), oracle.F32, p, s, b, oracle.F32, N, gs, bits)
    gate(y.cpu().numpy(), yref, "f32")


@pytest.mark.parametrize("bits", [2, 4, 6])
def test_transpose_false_awq_layout(bits):
    M, K, N, gs = 5, 96, 128, 64
    # W stored [K, N] quantized along N
    w, qw, (p, s, b) = _quant_pair(K, N, bits, gs, torch.bfloat16, 700 + bits)
    x = wl.gen_x(M, K, 701)
    y = api.qmm_matmul(x.to(DEV), qw, transpose=False, y_dtype=torch.float32)
    torch.cuda.synchronize()
    yref = oracle.matmul(np_storage(x), oracle.BF16, p, s, b, oracle.BF16, N, gs, bits, False)
    gate(y.cpu().numpy(), yref, "transpose=0")


def test_zero_rows_is_noop():
    qw = api.qmm_quantize(wl.gen_weight(64, 128, 1).to(DEV), 64, 4, torch.bfloat16)
    x = torch.empty(0, 128, dtype=torch.bfloat16, device=DEV)
    y = api.qmm_matmul(x, qw)
    assert tuple(y.shape) == (0, 64)


# ------------------------------------------------------------------ full-size decode and sweep
# Every output element of every full-size call is compared with the oracle;
# outputs sit in poisoned buffers with guard bands; the quantizer is checked
# bit for bit on every row.
@pytest.mark.parametrize("case", wl.WORKLOADS.decode, ids=lambda c: c.name)
def test_decode_full_size(case):
    w = wl.gen_weight(case.N, case.K, case.seed)
    x = wl.gen_x(case.M, case.K, case.seed + 1)
    qw = api.qmm_quantize(w.to(DEV), case.group_size, case.bits, torch.bfloat16)
    g32, g16 = Guarded((case.M, case.N), torch.float32), Guarded((case.M, case.N), torch.bfloat16)
    api.qmm_matmul(x.to(DEV), qw, True, out=g32.out)
    api.qmm_matmul(x.to(DEV), qw, True, out=g16.out)
    torch.cuda.synchronize()
    y32, y16 = g32.check(case.name), g16.check(case.name)
    p, s, b = qweight_np(qw)
    pr, sr, br = oracle.quantize(w.numpy(), oracle.F32, case.group_size, case.bits, oracle.BF16)
    assert np.array_equal(p, pr) and np.array_equal(s, sr) and np.array_equal(b, br)
    yref = oracle.matmul(np_storage(x), oracle.BF16, p, s, b, oracle.BF16, case.N,
                         case.group_size, case.bits)
    gate(y32.cpu().numpy(), yref, case.name)
    rne_equal(y16, y32)


_SWEEP_W = {}


def _sweep_weight(bits, gs, seed):
    """8192 x 8192 weights quantized once per (bits, group size); reused over M."""
    key = (bits, gs)
    if key not in _SWEEP_W:
        _SWEEP_W.clear()  # hold one matrix at a time
        w = wl.gen_weight(8192, 8192, seed)
        qw = api.qmm_quantize(w.to(DEV), gs, bits, torch.bfloat16)
        torch.cuda.synchronize()
        p, s, b = qweight_np(qw)
        pr, sr, br = oracle.quantize(w.numpy(), oracle.F32, gs, bits, oracle.BF16)
        assert np.array_equal(p, pr) and np.array_equal(s, sr) and np.array_equal(b, br)
        _SWEEP_W[key] = (w, qw, (p, s, b))
    return _SWEEP_W[key]


@pytest.mark.parametrize("case", wl.WORKLOADS.sweep, ids=lambda c: c.name)
def test_sweep_full_size(case):
    """Bit-width sweep at full size (N = K = 8192, b in {2,3,6,8}, gs in
    {32,64,128}, M in {1,4,16}): every output against the oracle, 16-bit
    output = RNE of the fp32 output, quantizer bit-exact on every row."""
    w, qw, (p, s, b) = _sweep_weight(case.bits, case.group_size, 2000 + 100 * case.bits + case.group_size)
    x = wl.gen_x(case.M, case.K, case.seed + 1)
    g32, g16 = Guarded((case.M, case.N), torch.float32), Guarded((case.M, case.N), torch.bfloat16)
    api.qmm_matmul(x.to(DEV), qw, True, out=g32.out)
    api.qmm_matmul(x.to(DEV), qw, True, out=g16.out)
    torch.cuda.synchronize()
    y32, y16 = g32.check(case.name), g16.check(case.name)
    yref = oracle.matmul(np_storage(x), oracle.BF16, p, s, b, oracle.BF16, case.N,
                         case.group_size, case.bits)
    gate(y32.cpu().numpy(), yref, case.name)
    rne_equal(y16, y32)


@pytest.mark.parametrize("M", [1, 4, 32])
def test_quantize_then_matmul_back_to_back(M):
    """The weights are rewritten by qmm_quantize immediately before qmm_matmul
    on the same stream, with no synchronization in between: the matmul must
    see the new weights (its kernels read nothing before the previous kernel
    in the stream has completed)."""
    from weight_only_quantized_qmm_b200 import _lib
    N, K = 4096, 4096
    w1 = wl.gen_weight(N, K, 950).to(DEV)
    w2 = wl.gen_weight(N, K, 951).to(DEV)
    x = wl.gen_x(M, K, 952).to(DEV)
    qw = api.qmm_quantize(w1, 64, 4, torch.bfloat16)
    api.qmm_matmul(x, qw, True, torch.float32)
    torch.cuda.synchronize()
    L = _lib.load()
    st = int(torch.cuda.current_stream().cuda_stream)
    y = torch.empty(M, N, dtype=torch.float32, device=DEV)
    rc = L.qmm_quantize(w2.data_ptr(), _lib.QMM_F32, N, K, 64, 4, _lib.QMM_BF16, qw.packed.data_ptr(),
                        qw.scales.data_ptr(), qw.biases.data_ptr(), st)
    assert rc == 0
    api.qmm_matmul(x, qw, True, out=y)
    torch.cuda.synchronize()
    p, s, b = oracle.quantize(w2.cpu().numpy(), oracle.F32, 64, 4, oracle.BF16)
    assert np.array_equal(packed_np(qw.packed), p)
    yref = oracle.matmul(np_storage(x.cpu()), oracle.BF16, p, s, b, oracle.BF16, N, 64, 4)
    gate(y.cpu().numpy(), yref, f"quantize->matmul M{M}")


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_gemv_activation_dynamic_range(bits, M, dtype):
    """Activations whose magnitude changes by many orders from group to group
    (and inside a group), all-zero groups and single-spike groups: the decode
    kernels carry x per group with its own power-of-two range, so every group
    keeps its precision whatever its neighbours' magnitude."""
    N, K, gs = 192, 4096, 64
    w, qw, (p, s, b) = _quant_pair(N, K, bits, gs, dtype, 1300 + bits + M)
    g = torch.Generator().manual_seed(1301 + M)
    # magnitudes stay inside the activation dtype's finite range (f16: < 6.5e4)
    lim, inner = (30, 3) if dtype == torch.bfloat16 else (2, 1)
    mag = 10.0 ** torch.randint(-lim, lim + 1, (M, K // gs), generator=g).double()
    x = (torch.randn(M, K, generator=g, dtype=torch.float64).clamp(-5, 5) * mag.repeat_interleave(gs, dim=1))
    x[:, 3 * gs:4 * gs] = 0.0                       # an all-zero group
    x[:, 5 * gs:6 * gs] = 0.0
    x[:, 5 * gs + 17] = 3.0                         # a single spike
    x[0, 7 * gs:8 * gs] *= torch.logspace(-inner, inner, gs, dtype=torch.float64)  # range inside a group
    x = x.to(dtype)
    assert torch.isfinite(x).all()
    g32 = Guarded((M, N), torch.float32)
    api.qmm_matmul(x.to(DEV), qw, True, out=g32.out)
    torch.cuda.synchronize()
    y = g32.check("y32")
    yref = oracle.matmul(np_storage(x), ORC[dtype], p, s, b, ORC[dtype], N, gs, bits)
    gate(y.cpu().numpy(), yref, f"dynamic range b{bits} M{M}")


@pytest.mark.parametrize("bits,gs,M,N,K", [(4, 64, 1, 4096, 4096), (4, 64, 1, 2048, 14336), (4, 64, 5, 2368, 4096),
                                           (4, 64, 16, 1024, 4096), (2, 128, 1, 2048, 8192), (3, 64, 1, 2048, 4096),
                                           (6, 64, 3, 2048, 4096), (8, 32, 1, 2048, 4096)])
def test_gemv_chained_through_x(bits, gs, M, N, K):
    """A GEMV whose x is the output of the GEMV launched just before it on the
    stream.  The first one lets its dependents launch early (programmatic
    dependent launch, after its plan barrier), so the second one runs its
    prologue and L2 prefetches while the first one still writes x: x must be
    read only after the first one completes.  Same bits as a call made after
    a synchronize."""
    seed = 1200 + 10 * bits + M
    _, qa, _ = _quant_pair(K, 1024, 4, 64, torch.bfloat16, seed)       # writes x: [M, K]
    _, qb, _ = _quant_pair(N, K, bits, gs, torch.bfloat16, seed + 1)
    xa = wl.gen_x(M, 1024, seed + 2).to(DEV)
    x = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
    ys = []
    for _ in range(3):
        x.zero_()
        api.qmm_matmul(xa, qa, True, out=x)
        ys.append(api.qmm_matmul(x, qb, True, torch.float32))
    torch.cuda.synchronize()
    yref = api.qmm_matmul(x, qb, True, torch.float32)
    torch.cuda.synchronize()
    for y in ys:
        assert torch.equal(y, yref)
