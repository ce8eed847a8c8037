"""GPU checks of the fused multi-part projection (qmm_matmul_parts): each
part's columns of y are exactly what qmm_matmul writes for that part alone
(the same kernel, only the output row stride differs), and within the
matmul tolerance of the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import Guarded, gate, np_storage, qweight_np
from tests.test_gpu_microscaled import mx_case
from weight_only_quantized_qmm_b200 import _lib, api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


def parts_for(K, seed):
    """q / k / v style parts of different kinds sharing K: 4-bit g64,
    4-bit g128, 6-bit g32, 8-bit g64, and an mxfp4 part"""
    specs = [(256, 64, 4), (128, 128, 4), (128, 32, 6), (72, 64, 8)]
    parts = []
    for i, (n, gs, bits) in enumerate(specs):
        parts.append(api.qmm_quantize(wl.gen_weight(n, K, seed + i).to(DEV), gs, bits, torch.bfloat16))
    parts.append(mx_case(oracle.MODE_MXFP4, 96, K, seed + 9)[0])
    return parts


@pytest.mark.parametrize("M", [1, 4, 16, 40, 300])
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32])
def test_parts_equal_single_calls(M, y_dtype):
    K = 1024
    parts = parts_for(K, 100 + M)
    x = wl.gen_x(M, K, 7 + M).to(DEV)
    ntot = sum(p.rows for p in parts)
    g = Guarded((M, ntot), y_dtype)
    api.qmm_matmul_parts(x, parts, out=g.out)
    torch.cuda.synchronize()
    y = g.check("parts")
    off = 0
    for p in parts:
        single = api.qmm_matmul(x, p, True, y_dtype=y_dtype)
        torch.cuda.synchronize()
        assert torch.equal(y[:, off:off + p.rows].view(torch.int16 if y_dtype != torch.float32 else torch.int32),
                           single.view(torch.int16 if y_dtype != torch.float32 else torch.int32)), \
            f"part rows {off}..{off + p.rows} differ from the single call"
        off += p.rows


@pytest.mark.parametrize("M", [1, 40])
def test_parts_against_oracle(M):
    K = 512
    parts = parts_for(K, 300 + M)
    x = wl.gen_x(M, K, 9 + M)
    y = api.qmm_matmul_parts(x.to(DEV), parts, y_dtype=torch.float32)
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    xs = np_storage(x)
    off = 0
    for i, p in enumerate(parts):
        if p.mode == api.QMM_MODE_AFFINE:
            packed, s, b = qweight_np(p)
            yref = oracle.matmul(xs, oracle.BF16, packed, s, b, oracle.BF16, p.rows, p.group_size, p.bits, True)
        else:
            yref = oracle.matmul_mx(xs, oracle.BF16, p.packed.cpu().numpy().view(np.uint32),
                                    p.scales.cpu().numpy(), p.mode, p.rows)
        gate(y[:, off:off + p.rows], yref, f"parts M{M} part{i}")
        off += p.rows


def test_parts_rejects_mismatched_input_dim():
    parts = [api.qmm_quantize(wl.gen_weight(64, 512, 1).to(DEV), 64, 4, torch.bfloat16),
             api.qmm_quantize(wl.gen_weight(64, 256, 2).to(DEV), 64, 4, torch.bfloat16)]
    x = wl.gen_x(1, 512, 3).to(DEV)
    with pytest.raises(_lib.QmmError):
        api.qmm_matmul_parts(x, parts)
