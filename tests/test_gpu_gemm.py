"""GPU parity of the prefill-shaped (M > 16) tcgen05 tensor-core GEMM against
the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import ORC, Guarded, gate, np_storage, qweight_np, rne_equal
from weight_only_quantized_qmm_b200 import api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
DTS = {torch.bfloat16: "bf16", torch.float16: "f16"}


def _case(M, N, K, bits, gs, dtype, seed):
    """fp32 and 16-bit outputs in poisoned buffers with guard bands."""
    w = wl.gen_weight(N, K, seed)
    qw = api.qmm_quantize(w.to(DEV), gs, bits, dtype)
    x = wl.gen_x(M, K, seed + 1, DTS[dtype])
    g32, g16 = Guarded((M, N), torch.float32), Guarded((M, N), dtype)
    api.qmm_matmul(x.to(DEV), qw, True, out=g32.out)
    api.qmm_matmul(x.to(DEV), qw, True, out=g16.out)
    torch.cuda.synchronize()
    return x, qw, g32.check("y32"), g16.check("y16")


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


def _tile_cover(n, tile, per_tile, rng):
    """per_tile distinct indices in every tile of `tile` along [0, n), always
    including the first and last index of each tile"""
    out = []
    for t0 in range(0, n, tile):
        t1 = min(n, t0 + tile)
        pick = {t0, t1 - 1}
        while len(pick) < min(per_tile, t1 - t0):
            pick.add(int(rng.integers(t0, t1)))
        out.extend(sorted(pick))
    return np.array(out)


@pytest.mark.parametrize("case", wl.WORKLOADS.prefill, ids=lambda c: c.name)
def test_prefill_full_size(case):
    """Every output of the GEMM against the oracle's dequantized weights in an
    fp64 library GEMM (oracle.matmul_dense); in addition the plain oracle
    loops check 2 tokens of every 256-token tile and 2 weight rows of every
    128-row tile; the whole 16-bit output equals RNE of the fp32 output;
    every output written, guard bands intact (poisoned buffers)."""
    x, qw, y32, y16 = _case(case.M, case.N, case.K, case.bits, case.group_size, torch.bfloat16,
                            case.seed)
    p, s, b = qweight_np(qw)
    xs = np_storage(x)
    y = y32.cpu().numpy()
    ref = oracle.matmul_dense(xs, oracle.BF16, p, s, b, oracle.BF16, case.N, case.group_size,
                              case.bits)
    gate(y, ref, case.name + " all outputs")
    del ref
    rng = np.random.default_rng(case.seed)
    toks = _tile_cover(case.M, 256, 2, rng)
    ref_t = oracle.matmul(xs[toks], oracle.BF16, p, s, b, oracle.BF16, case.N, case.group_size,
                          case.bits)
    gate(y[toks], ref_t, case.name + " token rows")
    rows = _tile_cover(case.N, 128, 2, rng)
    ref_r = oracle.matmul(xs, oracle.BF16, p[rows], s[rows], b[rows], oracle.BF16, len(rows),
                          case.group_size, case.bits)
    gate(y[:, rows], ref_r, case.name + " weight rows")
    rne_equal(y16, y32)
