"""The allocation-free MoE prefill entry point (qmm_moe_gemm_id_noalloc) gives
the same results as the routing + GEMM pair that uses a caller workspace.

It exists for callers that cannot provide device memory (an operator or
plugin interface that only hands over its inputs and outputs, or a path on
which cudaMalloc is not allowed); its schedule lives in a fixed scratch array
inside the library.  Two calls in a row, with different routing and
activations, must each match the workspace path: the second call sees the
first call's leftovers in the shared scratch and must not depend on them.
This file is collected last, so that a run stopping at its first failure has
run every other test before it."""
import pytest
import torch

from tests.helpers import gate
from weight_only_quantized_qmm_b200 import _lib, api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _stack(E, n_rows, n_cols, seed):
    qw = api.qmm_quantize(wl.gen_weight(E * n_rows, n_cols, seed).to(DEV), 64, 4, torch.bfloat16)
    return api.ExpertStack.from_qweight(qw, E)


def _with_workspace(a, ids, batch, top_k, ne11, st, E):
    ws = api.moe_workspace(batch * top_k, E)
    api.qmm_moe_compute_ids_tpe(ids, E, ws)
    return api.qmm_moe_gemm_id(a, batch, top_k, ne11, ws, st, torch.float32)


def test_noalloc_matches_the_workspace_path_on_two_calls_in_a_row():
    E, n_rows, n_cols, top_k = 64, 256, 512, 4
    st = _stack(E, n_rows, n_cols, 990)
    for call, (batch, ne11) in enumerate([(300, 1), (97, top_k)]):  # different sizes and routing
        ids = wl.gen_moe_ids(batch, E, top_k, 991 + call).to(DEV)
        a = wl.gen_x(batch * ne11, n_cols, 993 + call).to(DEV)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        got = api.qmm_moe_gemm_id_noalloc(a, ids, batch, top_k, ne11, st, torch.float32, d_status=status)
        ref = _with_workspace(a, ids, batch, top_k, ne11, st, E)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.isfinite(got).all()
        gate(got.cpu().numpy(), ref.cpu().numpy(), f"no-alloc call {call + 1}")


def test_noalloc_rejects_calls_beyond_its_scratch():
    E, top_k = 300, 2  # more experts than the scratch is sized for
    st = _stack(E, 64, 256, 995)
    ids = wl.gen_moe_ids(8, E, top_k, 996).to(DEV)
    a = wl.gen_x(8, 256, 997).to(DEV)
    with pytest.raises(_lib.QmmError) as e:
        api.qmm_moe_gemm_id_noalloc(a, ids, 8, top_k, 1, st)
    assert e.value.code == _lib.QMM_ERR_UNSUPPORTED
    st = _stack(8, 64, 256, 998)
    big = torch.zeros(8193 * 2, dtype=torch.int32, device=DEV)  # 16386 pairs
    with pytest.raises(_lib.QmmError) as e:
        api.qmm_moe_gemm_id_noalloc(wl.gen_x(8193, 256, 999).to(DEV), big, 8193, 2, 1, st)
    assert e.value.code == _lib.QMM_ERR_UNSUPPORTED
