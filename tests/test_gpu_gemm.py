"""GPU parity of the prefill-shaped (M > 16) tcgen05 tensor-core GEMM against
the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import ORC, gate, np_storage, qweight_np, rne_equal
from weight_only_quantized_qmm_b200 import api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
DTS = {torch.bfloat16: "bf16", torch.float16: "f16"}


def _case(M, N, K, bits, gs, dtype, seed):
    w = wl.gen_weight(N, K, seed)
    qw = api.qmm_quantize(w.to(DEV), gs, bits, dtype)
    x = wl.gen_x(M, K, seed + 1, DTS[dtype])
    y32 = api.qmm_matmul(x.to(DEV), qw, True, torch.float32)
    y16 = api.qmm_matmul(x.to(DEV), qw, True, dtype)
    torch.cuda.synchronize()
    return x, qw, y32, y16


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_gemm_widths_and_groups(bits, gs):
    M, N, K = 40, 160, 2 * 128
    x, qw, y32, y16 = _case(M, N, K, bits, gs, torch.bfloat16, 10 + bits + gs)
    p, s, b = qweight_np(qw)
    yref = oracle.matmul(np_storage(x), oracle.BF16, p, s, b, oracle.BF16, N, gs, bits)
    gate(y32.cpu().numpy(), yref, f"gemm b{bits} g{gs}")
    rne_equal(y16, y32)


@pytest.mark.parametrize("M,N,K", [(17, 128, 64), (256, 256, 512), (300, 200, 384), (513, 129, 96)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_gemm_tiles_and_ragged_edges(M, N, K, dtype):
    gs = 32 if K % 64 else 64
    x, qw, y32, y16 = _case(M, N, K, 4, gs, dtype, 100 + M + N)
    p, s, b = qweight_np(qw)
    yref = oracle.matmul(np_storage(x), ORC[dtype], p, s, b, ORC[dtype], N, gs, 4)
    gate(y32.cpu().numpy(), yref, f"M{M} N{N} K{K}")
    rne_equal(y16, y32)


def test_gemm_weight_operand_equals_bf16_dequant():
    """the GEMM's weight operand is the bf16 rounding of q*s + b: with x a
    one-hot row the output is exactly the dequantized weight column"""
    N, K = 256, 256
    w = wl.gen_weight(N, K, 7)
    qw = api.qmm_quantize(w.to(DEV), 64, 4, torch.bfloat16)
    x = torch.zeros(32, K, dtype=torch.bfloat16)
    for i in range(32):
        x[i, 5 * i] = 1.0
    y = api.qmm_matmul(x.to(DEV), qw, True, torch.float32)
    deq = api.qmm_dequantize(qw, torch.bfloat16).float()
    torch.cuda.synchronize()
    for i in range(32):
        assert torch.equal(y[i].cpu(), deq[:, 5 * i].cpu())


@pytest.mark.parametrize("case", wl.WORKLOADS.prefill, ids=lambda c: c.name)
def test_prefill_full_size_sampled(case):
    x, qw, y32, y16 = _case(case.M, case.N, case.K, case.bits, case.group_size, torch.bfloat16,
                            case.seed)
    p, s, b = qweight_np(qw)
    rng = np.random.default_rng(case.seed)
    ms = np.concatenate([rng.integers(0, case.M, 300), [0, case.M - 1]])
    ns = np.concatenate([rng.integers(0, case.N, 300), [case.N - 1, 0]])
    coords = list(zip(ms.tolist(), ns.tolist()))
    yref = oracle.matmul_elements(np_storage(x), oracle.BF16, p, s, b, oracle.BF16, case.N,
                                  case.group_size, case.bits, coords)
    got = y32.cpu().numpy()[ms, ns]
    gate(got, yref, case.name)
    # bf16 output: the same kernel's fp32 result rounded once
    idx = torch.tensor(ms), torch.tensor(ns)
    assert torch.equal(y16.cpu()[idx].view(torch.int16), y32.cpu()[idx].to(torch.bfloat16).view(torch.int16))
    assert torch.isfinite(y16).all()
