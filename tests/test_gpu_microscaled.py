"""GPU parity of the microscaled modes (mxfp4, mxfp8, nvfp4): standalone
dequantization bit for bit, and the matmul within the matmul tolerance,
against the CPU oracle through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import ORC, Guarded, gate, np_storage, rne_equal
from weight_only_quantized_qmm_b200 import api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
MODES = [oracle.MODE_MXFP4, oracle.MODE_MXFP8, oracle.MODE_NVFP4]


def mx_case(mode, rows, cols, seed, full_range=False):
    """random lanes (every code, the +-480 bytes of E4M3 included) and scale
    bytes of the kind the quantizers emit (E8M0 near 2^-7; positive E4M3)"""
    bits, gs = oracle.MX_PARAMS[mode]
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 1 << bits, (rows, cols), dtype=np.uint8)
    if mode == oracle.MODE_NVFP4:
        sc = rng.integers(0x01, 0x7F, (rows, cols // gs), dtype=np.uint8)
    else:
        lo, hi = (1, 255) if full_range else (112, 128)
        sc = rng.integers(lo, hi, (rows, cols // gs), dtype=np.uint8)
    packed = np.stack([oracle.pack_row(r, bits) for r in codes])
    qw = api.mx_qweight(torch.from_numpy(packed.view(np.int32)).to(DEV), torch.from_numpy(sc).to(DEV), mode,
                        rows, cols)
    return qw, packed, sc


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_dequant_mx_bit_exact(mode, out_dtype):
    qw, packed, sc = mx_case(mode, 23, 256, 10 + mode, full_range=out_dtype == torch.float32)
    g = Guarded((23, 256), out_dtype)
    api.qmm_dequantize(qw, out=g.out)
    torch.cuda.synchronize()
    out = g.check("dequant mx")
    ref = oracle.dequantize_mx(packed, sc, mode, 256, ORC[out_dtype])
    assert np.array_equal(np_storage(out), ref)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [1, 5, 16, 40])
@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_matmul_mx(mode, M, x_dtype):
    N, K = 144, 512
    qw, packed, sc = mx_case(mode, N, K, 30 + mode + M)
    x = wl.gen_x(M, K, 31 + M, {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[x_dtype])
    g32, gx = Guarded((M, N), torch.float32), Guarded((M, N), x_dtype)
    api.qmm_matmul(x.to(DEV), qw, True, out=g32.out)
    api.qmm_matmul(x.to(DEV), qw, True, out=gx.out)
    torch.cuda.synchronize()
    y32, yx = g32.check("mx y32"), gx.check("mx y")
    yref = oracle.matmul_mx(np_storage(x), ORC[x_dtype], packed, sc, mode, N)
    gate(y32.cpu().numpy(), yref, f"mx mode {mode} M{M}")
    # the output in the activation dtype is the same result rounded once
    rne_equal(yx, y32)


def test_matmul_mx_decode_shape():
    """a decode-sized mxfp4 call (14336 x 4096, one token)"""
    N, K = 14336, 4096
    qw, packed, sc = mx_case(oracle.MODE_MXFP4, N, K, 77)
    x = wl.gen_x(1, K, 78)
    g = Guarded((1, N), torch.float32)
    api.qmm_matmul(x.to(DEV), qw, True, out=g.out)
    torch.cuda.synchronize()
    yref = oracle.matmul_mx(np_storage(x), oracle.BF16, packed, sc, oracle.MODE_MXFP4, N)
    gate(g.check("mx decode").cpu().numpy(), yref, "mxfp4 decode 14336x4096")
