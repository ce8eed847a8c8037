"""GPU parity of the per-tensor dynamic-range int8 calls against the CPU
oracle through the C ABI: quantize (codes and params) and dequantize bit for
bit, the matmul within the matmul tolerance."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import ORC, Guarded, gate, np_storage, rne_equal
from weight_only_quantized_qmm_b200 import api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
_NAME = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}


def weights(n, k, seed, dtype=torch.float32, std=0.02):
    return wl.gen_weight(n, k, seed, std).to(dtype)


@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", [(7,), (1, 4099), (256, 512), (3072, 768)])
def test_quantize_bit_exact(w_dtype, shape):
    n = int(np.prod(shape))
    w = weights(1, n, 3 + n, w_dtype).reshape(shape)
    q, params = api.qmm_quantize_dynamic_int8(w.to(DEV))
    torch.cuda.synchronize()
    q_ref, p_ref = oracle.quantize_dynamic_int8(np_storage(w).reshape(-1), ORC[w_dtype])
    assert params.cpu().numpy().tolist() == p_ref.tolist()
    assert np.array_equal(q.cpu().numpy().reshape(-1), q_ref)


def test_quantize_special_values():
    """NaN elements are passed over by min/max and get code 0; a constant
    tensor takes the FLT_EPSILON scale (all codes -128); an exact page case"""
    cases = [np.array([0.5, np.nan, -1.0, 2.0, np.nan, 0.0] * 50, dtype=np.float32),
             np.full(333, 0.625, dtype=np.float32),
             np.array([-2.0, -1.0, 0.0, 0.5, 1.0, 2.0, 3.5], dtype=np.float32)]
    for w in cases:
        q, params = api.qmm_quantize_dynamic_int8(torch.from_numpy(w).to(DEV))
        torch.cuda.synchronize()
        q_ref, p_ref = oracle.quantize_dynamic_int8(w, oracle.F32)
        assert params.cpu().numpy().tolist() == p_ref.tolist()
        assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n", [5, 4096, 4099, 1 << 20])
def test_dequant_bit_exact(out_dtype, n):
    rng = np.random.default_rng(n)
    q = rng.integers(-128, 128, n, dtype=np.int8)
    params = np.array([-0.07, 0.05, -0.071, 0.0493], dtype=np.float32)  # output range used
    g = Guarded((n,), out_dtype)
    api.qmm_dequantize_dynamic_int8(torch.from_numpy(q).to(DEV), torch.from_numpy(params).to(DEV), out=g.out)
    torch.cuda.synchronize()
    out = g.check("dequant int8")
    ref = oracle.dequantize_dynamic_int8(q, params, ORC[out_dtype])
    assert np.array_equal(np_storage(out), ref)


@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("M", [1, 3, 8, 13, 40])
@pytest.mark.parametrize("K", [512, 1000, 4096])
def test_matmul(x_dtype, M, K):
    """K = 1000 takes the unvectorised row walk (K % 16 != 0)"""
    N = 200
    w = weights(N, K, 40 + K)
    q, params = api.qmm_quantize_dynamic_int8(w.to(DEV))
    x = wl.gen_x(M, K, 41 + M, _NAME[x_dtype])
    g32, gx = Guarded((M, N), torch.float32), Guarded((M, N), x_dtype)
    api.qmm_matmul_dynamic_int8(x.to(DEV), q, params, out=g32.out)
    api.qmm_matmul_dynamic_int8(x.to(DEV), q, params, out=gx.out)
    torch.cuda.synchronize()
    y32, yx = g32.check("int8 y32"), gx.check("int8 y")
    yref = oracle.matmul_dynamic_int8(np_storage(x), ORC[x_dtype], q.cpu().numpy(), params.cpu().numpy())
    gate(y32.cpu().numpy(), yref, f"dynamic int8 M{M} K{K}")
    rne_equal(yx, y32)


def test_matmul_long_rows_read_x_from_global():
    """rows too long to stage x in shared memory"""
    M, N, K = 2, 64, 65536
    w = weights(N, K, 50)
    q, params = api.qmm_quantize_dynamic_int8(w.to(DEV))
    x = wl.gen_x(M, K, 51)
    g = Guarded((M, N), torch.float32)
    api.qmm_matmul_dynamic_int8(x.to(DEV), q, params, out=g.out)
    torch.cuda.synchronize()
    yref = oracle.matmul_dynamic_int8(np_storage(x), oracle.BF16, q.cpu().numpy(), params.cpu().numpy())
    gate(g.check("int8 long").cpu().numpy(), yref, "dynamic int8 K65536")


def test_matmul_decode_shape_all_outputs():
    """a decode-sized call (4096 x 4096, one token), every output compared"""
    N, K = 4096, 4096
    w = weights(N, K, 60)
    q, params = api.qmm_quantize_dynamic_int8(w.to(DEV))
    x = wl.gen_x(1, K, 61)
    g32, g16 = Guarded((1, N), torch.float32), Guarded((1, N), torch.bfloat16)
    api.qmm_matmul_dynamic_int8(x.to(DEV), q, params, out=g32.out)
    api.qmm_matmul_dynamic_int8(x.to(DEV), q, params, out=g16.out)
    torch.cuda.synchronize()
    yref = oracle.matmul_dynamic_int8(np_storage(x), oracle.BF16, q.cpu().numpy(), params.cpu().numpy())
    y32 = g32.check("int8 decode")
    gate(y32.cpu().numpy(), yref, "dynamic int8 decode 4096x4096")
    rne_equal(g16.check("int8 decode bf16"), y32)


@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("N,K", [(200, 2048), (1000, 14336)])
def test_matmul_streaming_kernel_shapes(x_dtype, M, N, K):
    """few tokens, 16-bit x and K a multiple of 512: the streaming tensor-core
    GEMV with the per-tensor scale (K = 14336: 224 groups, a partial last
    unit; N = 200: a ragged last row tile); every output compared"""
    w = weights(N, K, 70 + K + M)
    q, params = api.qmm_quantize_dynamic_int8(w.to(DEV))
    x = wl.gen_x(M, K, 71 + M, _NAME[x_dtype])
    g32, gx = Guarded((M, N), torch.float32), Guarded((M, N), x_dtype)
    api.qmm_matmul_dynamic_int8(x.to(DEV), q, params, out=g32.out)
    api.qmm_matmul_dynamic_int8(x.to(DEV), q, params, out=gx.out)
    torch.cuda.synchronize()
    y32, yx = g32.check("int8 stream y32"), gx.check("int8 stream y")
    yref = oracle.matmul_dynamic_int8(np_storage(x), ORC[x_dtype], q.cpu().numpy(), params.cpu().numpy())
    gate(y32.cpu().numpy(), yref, f"dynamic int8 stream M{M} {N}x{K}")
    rne_equal(yx, y32)
