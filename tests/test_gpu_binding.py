"""The binding keeps a QWeight's validated state between calls; a weight
tensor that is replaced, shrunk or retyped after a successful call is checked
again (ValueError, nothing launched), and the restored weight computes the
same result as before."""
import pytest
import torch

from weight_only_quantized_qmm_b200 import api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_changed_weight_tensors_are_checked_again():
    N, K = 256, 512
    qw = api.qmm_quantize(wl.gen_weight(N, K, 31).to(DEV), 64, 4, torch.bfloat16)
    x = wl.gen_x(2, K, 32).to(DEV)
    y0 = api.qmm_matmul(x, qw, y_dtype=torch.float32)
    torch.cuda.synchronize()
    packed, scales, biases = qw.packed, qw.scales, qw.biases

    qw.packed = packed[: N // 2].clone()  # too few rows
    with pytest.raises(ValueError, match="packed holds"):
        api.qmm_matmul(x, qw)
    qw.packed = packed

    qw.scales = scales.to(torch.float16)  # retyped: no longer the biases' dtype
    with pytest.raises(ValueError, match="biases has dtype"):
        api.qmm_matmul(x, qw)
    qw.scales = scales

    qw.biases = biases.reshape(-1)[: biases.numel() - 1].clone()  # one element short
    with pytest.raises(ValueError, match="biases holds"):
        api.qmm_matmul(x, qw)
    qw.biases = biases

    qw.rows = N + 16  # a stated shape the tensors do not hold
    with pytest.raises(ValueError, match="holds"):
        api.qmm_matmul(x, qw)
    qw.rows = N

    y1 = api.qmm_matmul(x, qw, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)


def test_host_weights_are_refused_after_a_device_call():
    N, K = 128, 256
    qw = api.qmm_quantize(wl.gen_weight(N, K, 33).to(DEV), 64, 4, torch.bfloat16)
    x = wl.gen_x(1, K, 34).to(DEV)
    api.qmm_matmul(x, qw)
    torch.cuda.synchronize()
    qw.scales = qw.scales.cpu()
    qw.biases = qw.biases.cpu()
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.qmm_matmul(x, qw)


def test_changed_expert_stacks_are_checked_again():
    E, n_rows, n_cols, k = 8, 128, 256, 4
    q = api.qmm_quantize(wl.gen_weight(E * n_rows, n_cols, 35).to(DEV), 64, 4, torch.bfloat16)
    gate = api.ExpertStack.from_qweight(q, E)
    up = api.ExpertStack.from_qweight(
        api.qmm_quantize(wl.gen_weight(E * n_rows, n_cols, 36).to(DEV), 64, 4, torch.bfloat16), E)
    a = wl.gen_x(1, n_cols, 37).to(DEV).reshape(-1)
    ids = torch.tensor([0, 3, 5, 7], dtype=torch.int32, device=DEV)
    h0 = api.qmm_moe_gemv_id_gate_up_silu(a, ids, k, gate, up, out_dtype=torch.float32)
    torch.cuda.synchronize()
    scales = up.scales
    up.scales = scales.reshape(-1)[: scales.numel() - 1].clone()  # one element short
    with pytest.raises(ValueError, match="up.scales holds"):
        api.qmm_moe_gemv_id_gate_up_silu(a, ids, k, gate, up)
    up.scales = scales
    gate.num_experts = E + 1  # a stated size the tensors do not hold
    with pytest.raises(ValueError, match="holds"):
        api.qmm_moe_gemv_id_gate_up_silu(a, ids, k, gate, up)
    gate.num_experts = E
    h1 = api.qmm_moe_gemv_id_gate_up_silu(a, ids, k, gate, up, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(h0, h1)
