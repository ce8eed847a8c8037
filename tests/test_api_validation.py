"""The Python binding refuses, before calling the library, every argument that
would make a kernel read or write out of bounds: too-small outputs, weights
whose tensors do not match their stated shape, ids of the wrong dtype or
length, activations shorter than the last pair's row, non-contiguous or host
tensors.  No GPU is needed: the checks run before any device work (CPU
tensors reach the size, dtype and layout checks first)."""
import pytest
import torch

from weight_only_quantized_qmm_b200 import api


def qweight(rows=32, cols=128, bits=4, gs=64, **over):
    t = dict(packed=torch.zeros(rows, cols * bits // 32, dtype=torch.int32),
             scales=torch.zeros(rows, cols // gs, dtype=torch.bfloat16),
             biases=torch.zeros(rows, cols // gs, dtype=torch.bfloat16))
    t.update(over)
    return api.QWeight(t["packed"], t["scales"], t["biases"], rows, cols, gs, bits)


def stack(E=4, n_rows=16, n_cols=128, bits=4, gs=64, **over):
    q = qweight(E * n_rows, n_cols, bits, gs, **over)
    return api.ExpertStack(q.packed, q.scales, q.biases, E, n_rows, n_cols, gs, bits)


def raises(fn, match):
    with pytest.raises(ValueError, match=match):
        fn()


def test_valid_host_tensors_reach_the_device_check():
    x = torch.zeros(2, 128, dtype=torch.bfloat16)
    raises(lambda: api.qmm_matmul(x, qweight()), "CUDA tensor")


def test_weight_tensors_must_match_the_stated_shape():
    x = torch.zeros(2, 128, dtype=torch.bfloat16)
    raises(lambda: api.qmm_matmul(x, qweight(packed=torch.zeros(31, 16, dtype=torch.int32))),
           "packed holds")
    raises(lambda: api.qmm_matmul(x, qweight(scales=torch.zeros(32, 1, dtype=torch.bfloat16))),
           "scales holds")
    raises(lambda: api.qmm_matmul(x, qweight(biases=torch.zeros(32, 2, dtype=torch.float16))),
           "biases has dtype")
    raises(lambda: api.qmm_matmul(x, qweight(packed=torch.zeros(32, 16, dtype=torch.int64))),
           "packed has dtype")
    raises(lambda: api.qmm_matmul(x, qweight(packed=torch.zeros(16, 32, dtype=torch.int32).t())),
           "contiguous")


def test_matmul_output_checked():
    x = torch.zeros(2, 128, dtype=torch.bfloat16)
    raises(lambda: api.qmm_matmul(x, qweight(), out=torch.zeros(2, 31)), "out holds")
    raises(lambda: api.qmm_matmul(x, qweight(), out=torch.zeros(2, 33)), "expected 2x32")
    raises(lambda: api.qmm_matmul(x, qweight(), out=torch.zeros(2, 32, dtype=torch.int32)),
           "out has dtype")
    raises(lambda: api.qmm_matmul(x, qweight(), out=torch.zeros(32, 2).t()), "contiguous")


def test_dequantize_output_checked():
    raises(lambda: api.qmm_dequantize(qweight(), out=torch.zeros(32, 127)), "out holds")


def test_moe_ids_checked():
    a = torch.zeros(4 * 128, dtype=torch.bfloat16)
    st = stack()
    raises(lambda: api.qmm_moe_gemv_id(a, torch.zeros(4, dtype=torch.int64), 4, 128, st), "ids has dtype")
    raises(lambda: api.qmm_moe_gemv_id(a, torch.zeros(3, dtype=torch.int32), 4, 128, st), "ids holds")


def test_moe_activation_extent_checked():
    ids = torch.zeros(8, dtype=torch.int32)
    st = stack()
    # single: the last pair reads a[3*128 : 3*128 + 128]
    raises(lambda: api.qmm_moe_gemv_id(torch.zeros(4 * 128 - 1, dtype=torch.bfloat16), ids, 4, 128, st),
           "a holds")
    # batched: pair 7 of m=2, top_k=4 reads a[1*512 + 3*128 : ... + 128]
    raises(lambda: api.qmm_moe_gemv_id_batched(torch.zeros(1023, dtype=torch.bfloat16), ids, 2, 4, 512,
                                               128, st), "a holds")
    # fused: every pair reads a[0:128]
    raises(lambda: api.qmm_moe_gemv_id_gate_up_silu(torch.zeros(127, dtype=torch.bfloat16), ids, 8, st,
                                                    stack()), "a holds")


def test_moe_outputs_stacks_and_status_checked():
    a = torch.zeros(8 * 128, dtype=torch.bfloat16)
    ids = torch.zeros(8, dtype=torch.int32)
    st = stack()
    raises(lambda: api.qmm_moe_gemv_id(a, ids, 8, 128, st, out=torch.zeros(8, 15)), "out holds")
    raises(lambda: api.qmm_moe_gemv_id(a, ids, 8, 128, stack(packed=torch.zeros(63, 16, dtype=torch.int32))),
           "packed holds")
    raises(lambda: api.qmm_moe_gemv_id_gate_up_silu_batched(
        a, ids, 2, 4, 128, 0, st, stack(scales=torch.zeros(64, 1, dtype=torch.bfloat16))), "scales holds")
    raises(lambda: api.qmm_moe_gemv_id(a, ids, 8, 128, st, out=torch.zeros(8, 16),
                                       d_status=torch.zeros(1, dtype=torch.int64)), "d_status has dtype")
