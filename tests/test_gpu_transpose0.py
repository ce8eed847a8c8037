"""GPU parity of the [K, N] weight layout (quantized_matmul with transpose
false, the AWQ layout) against the CPU oracle: the few-token kernel for
whole-word codes (bits 2, 4, 8) and the general path for 3 and 6 bits, over
ragged column counts, row counts that span several staged chunks of x, and a
decode-sized call with every output compared."""
import pytest
import torch

import oracle
from tests.helpers import ORC, Guarded, gate, np_storage, qweight_np, rne_equal
from weight_only_quantized_qmm_b200 import api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
_NAME = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}


def case(K, N, bits, gs, dtype, seed):
    w = wl.gen_weight(K, N, seed).to(torch.float32)
    qw = api.qmm_quantize(w.to(DEV), gs, bits, dtype)  # stored [K, N], quantized along N
    torch.cuda.synchronize()
    return qw, qweight_np(qw)


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("M", [1, 3, 8, 16])
def test_transpose0_matches_oracle(bits, gs, M):
    K, N = 1500, 3 * 128 + (gs if gs < 128 else 128)  # K spans two staged chunks; N not a block multiple
    qw, (p, s, b) = case(K, N, bits, gs, torch.bfloat16, 900 + bits + gs + M)
    x = wl.gen_x(M, K, 901 + M)
    g32, g16 = Guarded((M, N), torch.float32), Guarded((M, N), torch.bfloat16)
    api.qmm_matmul(x.to(DEV), qw, transpose=False, out=g32.out)
    api.qmm_matmul(x.to(DEV), qw, transpose=False, out=g16.out)
    torch.cuda.synchronize()
    y32 = g32.check("t0 y32")
    yref = oracle.matmul(np_storage(x), oracle.BF16, p, s, b, oracle.BF16, N, gs, bits, False)
    gate(y32.cpu().numpy(), yref, f"transpose=0 b{bits} g{gs} M{M}")
    rne_equal(g16.check("t0 y16"), y32)


@pytest.mark.parametrize("x_dtype", [torch.float16, torch.float32])
def test_transpose0_other_dtypes(x_dtype):
    K, N, bits, gs = 700, 512, 4, 64
    qw, (p, s, b) = case(K, N, bits, gs, x_dtype, 950)
    x = wl.gen_x(5, K, 951, _NAME[x_dtype])
    y = api.qmm_matmul(x.to(DEV), qw, transpose=False, y_dtype=torch.float32)
    torch.cuda.synchronize()
    yref = oracle.matmul(np_storage(x), ORC[x_dtype], p, s, b, ORC[x_dtype], N, gs, bits, False)
    gate(y.cpu().numpy(), yref, f"transpose=0 {x_dtype}")


@pytest.mark.parametrize("N", [4096, 14336])
def test_transpose0_decode_size_all_outputs(N):
    K, bits, gs = 4096, 4, 64
    qw, (p, s, b) = case(K, N, bits, gs, torch.bfloat16, 960 + N)
    x = wl.gen_x(1, K, 961)
    g = Guarded((1, N), torch.float32)
    api.qmm_matmul(x.to(DEV), qw, transpose=False, out=g.out)
    torch.cuda.synchronize()
    yref = oracle.matmul(np_storage(x), oracle.BF16, p, s, b, oracle.BF16, N, gs, bits, False)
    gate(g.check("t0 decode").cpu().numpy(), yref, f"transpose=0 decode {K}x{N}")
