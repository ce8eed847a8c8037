"""GPU parity of the MoE indirect-dispatch GEMVs (single, batched, fused
gate+up+SiLU) against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import ORC, Guarded, gate, np_storage, qweight_np, rne_equal
from weight_only_quantized_qmm_b200 import api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


def make_stack(E, n_rows, n_cols, bits, gs, seed, dtype=torch.bfloat16):
    w = wl.gen_weight(E * n_rows, n_cols, seed)
    qw = api.qmm_quantize(w.to(DEV), gs, bits, dtype)
    torch.cuda.synchronize()
    p, s, b = qweight_np(qw)
    st = api.ExpertStack.from_qweight(qw, E)
    ost = oracle.Stack(p, s, b, ORC[dtype], E, n_rows, n_cols, gs, bits)
    return st, ost


@pytest.mark.parametrize("bits,gs", [(4, 64), (3, 32), (8, 128), (2, 64), (6, 64)])
def test_moe_gemv_id_single(bits, gs):
    E, n_rows, n_cols = 9, 80, 2 * gs * 2
    st, ost = make_stack(E, n_rows, n_cols, bits, gs, 10 + bits)
    n_sel, stride = 6, n_cols + 32
    a = wl.gen_x(1, stride * n_sel, 11).reshape(-1)
    ids = torch.tensor([3, 0, 8, 3, 5, 3], dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    g32, g16 = Guarded((n_sel, n_rows), torch.float32), Guarded((n_sel, n_rows), torch.bfloat16)
    api.qmm_moe_gemv_id(a.to(DEV), ids.to(DEV), n_sel, stride, st, out=g32.out, d_status=status)
    api.qmm_moe_gemv_id(a.to(DEV), ids.to(DEV), n_sel, stride, st, out=g16.out)
    torch.cuda.synchronize()
    out32, out16 = g32.check("moe"), g16.check("moe bf16")
    ref, rc = oracle.moe_gemv_id(np_storage(a), oracle.BF16, ids.numpy(), n_sel, stride, ost)
    assert rc == oracle.ORC_OK and int(status.item()) == 0
    gate(out32.cpu().numpy(), ref, f"moe b{bits}")
    rne_equal(out16, out32)


@pytest.mark.parametrize("m,top_k", [(3, 2), (5, 4), (20, 4)])
def test_moe_gemv_id_batched(m, top_k):
    E, n_rows, n_cols, bits, gs = 16, 64, 256, 4, 64
    st, ost = make_stack(E, n_rows, n_cols, bits, gs, 20 + m)
    outer, inner = top_k * n_cols, n_cols  # [m, top_k, n_cols] activations
    a = wl.gen_x(m * top_k, n_cols, 21).reshape(-1)
    ids = wl.gen_moe_ids(m, E, top_k, 22)
    g32 = Guarded((m * top_k, n_rows), torch.float32)
    api.qmm_moe_gemv_id_batched(a.to(DEV), ids.to(DEV), m, top_k, outer, inner, st, out=g32.out)
    torch.cuda.synchronize()
    out32 = g32.check("batched")
    ref, rc = oracle.moe_gemv_id_batched(np_storage(a), oracle.BF16, ids.numpy(), m, top_k, outer,
                                         inner, ost)
    assert rc == oracle.ORC_OK
    gate(out32.cpu().numpy(), ref, "batched")


@pytest.mark.parametrize("bits", [4, 8])
def test_moe_gate_up_silu(bits):
    E, n_rows, n_cols, gs = 12, 96, 512, 64
    g, og = make_stack(E, n_rows, n_cols, bits, gs, 30)
    u, ou = make_stack(E, n_rows, n_cols, bits, gs, 31)
    a = wl.gen_x(1, n_cols, 32).reshape(-1)
    ids = torch.tensor([7, 1, 11, 0, 4, 7, 2, 9], dtype=torch.int32)
    g32, g16 = Guarded((8, n_rows), torch.float32), Guarded((8, n_rows), torch.bfloat16)
    api.qmm_moe_gemv_id_gate_up_silu(a.to(DEV), ids.to(DEV), 8, g, u, out=g32.out)
    api.qmm_moe_gemv_id_gate_up_silu(a.to(DEV), ids.to(DEV), 8, g, u, out=g16.out)
    torch.cuda.synchronize()
    out32, out16 = g32.check("gate_up"), g16.check("gate_up bf16")
    ref, rc = oracle.moe_gate_up_silu(np_storage(a), oracle.BF16, ids.numpy(), 8, og, ou)
    assert rc == oracle.ORC_OK
    gate(out32.cpu().numpy(), ref, "gate_up_silu")
    rne_equal(out16, out32)


def test_moe_gate_up_silu_batched_many_tokens_per_expert():
    """more than 16 pairs on one expert: the kernel makes several token passes"""
    E, n_rows, n_cols, bits, gs = 4, 48, 256, 4, 64
    g, og = make_stack(E, n_rows, n_cols, bits, gs, 40)
    u, ou = make_stack(E, n_rows, n_cols, bits, gs, 41)
    m, top_k = 24, 2
    a = wl.gen_x(m, n_cols, 42).reshape(-1)
    ids = wl.gen_moe_ids(m, E, top_k, 43)
    out32 = api.qmm_moe_gemv_id_gate_up_silu_batched(a.to(DEV), ids.to(DEV), m, top_k, n_cols, 0,
                                                     g, u, torch.float32)
    torch.cuda.synchronize()
    ref, rc = oracle.moe_gate_up_silu_batched(np_storage(a), oracle.BF16, ids.numpy(), m, top_k,
                                              n_cols, 0, og, ou)
    assert rc == oracle.ORC_OK
    gate(out32.cpu().numpy(), ref, "batched gate_up_silu")


@pytest.mark.parametrize("dual", [False, True])
def test_moe_segments_split_one_expert_deterministic(dual):
    """Rows long enough for the streaming kernel (K = 2048) and ~12 pairs per
    expert, so an expert's pairs span several segments: every CTA must derive
    the same pair lists (outputs complete, identical between calls, 16-bit
    output = RNE of the fp32 output) and match the oracle."""
    E, n_rows, n_cols, bits, gs = 8, 64, 2048, 4, 64
    g, og = make_stack(E, n_rows, n_cols, bits, gs, 50)
    u, ou = make_stack(E, n_rows, n_cols, bits, gs, 51)
    m, top_k = 48, 2
    a = wl.gen_x(m, n_cols, 52).reshape(-1)
    ids = wl.gen_moe_ids(m, E, top_k, 53)
    assert int(torch.bincount(ids.reshape(-1), minlength=E).max()) > 8

    def call(dt):
        if dual:
            return api.qmm_moe_gemv_id_gate_up_silu_batched(a.to(DEV), ids.to(DEV), m, top_k, n_cols, 0,
                                                            g, u, dt)
        return api.qmm_moe_gemv_id_batched(a.to(DEV), ids.to(DEV), m, top_k, n_cols, 0, g, dt)

    outs = [call(torch.float32) for _ in range(3)]
    o16 = call(None)
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(outs[0], o)
    rne_equal(o16, outs[0])
    if dual:
        ref, rc = oracle.moe_gate_up_silu_batched(np_storage(a), oracle.BF16, ids.numpy(), m, top_k,
                                                  n_cols, 0, og, ou)
    else:
        ref, rc = oracle.moe_gemv_id_batched(np_storage(a), oracle.BF16, ids.numpy(), m, top_k,
                                             n_cols, 0, og)
    assert rc == oracle.ORC_OK
    gate(outs[0].cpu().numpy(), ref, "segments split")


def test_moe_bad_id_zero_row_and_status():
    E, n_rows, n_cols, bits, gs = 3, 32, 128, 4, 64
    st, ost = make_stack(E, n_rows, n_cols, bits, gs, 50)
    a = wl.gen_x(1, n_cols, 51).reshape(-1)
    ids = torch.tensor([1, 7, -2, 0], dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.full((4, n_rows), float("nan"), device=DEV)
    api.qmm_moe_gemv_id(a.to(DEV), ids.to(DEV), 4, 0, st, out=out, d_status=status)
    torch.cuda.synchronize()
    ref, rc = oracle.moe_gemv_id(np_storage(a), oracle.BF16, ids.numpy(), 4, 0, ost)
    assert rc == oracle.ORC_ERR_ID
    assert int(status.item()) & 7 == 7  # QMM_ERR_BAD_EXPERT_ID
    o = out.cpu().numpy()
    assert np.all(o[1] == 0) and np.all(o[2] == 0)
    gate(o[[0, 3]], ref[[0, 3]], "valid pairs")


@pytest.mark.parametrize("case", wl.WORKLOADS.moe, ids=lambda c: c.name)
def test_moe_config_full_size(case):
    """128 experts, gate/up [768 x 2048], down [2048 x 768], top-8, T tokens:
    fused gate+up+SiLU then down (src1_stride = 768).  Every output of every
    pair of both calls is compared with the oracle; outputs sit in poisoned
    buffers with guard bands."""
    E, dff, dm = case.num_experts, case.d_ff, case.d_model
    gate_s, og = make_stack(E, dff, dm, case.bits, case.group_size, case.seed)
    up_s, ou = make_stack(E, dff, dm, case.bits, case.group_size, case.seed + 1)
    down_s, od = make_stack(E, dm, dff, case.bits, case.group_size, case.seed + 2)
    T, k = case.tokens, case.top_k
    a = wl.gen_x(T, dm, case.seed + 3)
    ids = wl.gen_moe_ids(T, E, k, case.seed + 4)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gh, gh16 = Guarded((T * k, dff), torch.float32), Guarded((T * k, dff), torch.bfloat16)
    go = Guarded((T * k, dm), torch.float32)
    api.qmm_moe_gemv_id_gate_up_silu_batched(a.to(DEV).reshape(-1), ids.to(DEV), T, k, dm, 0,
                                             gate_s, up_s, out=gh.out, d_status=status)
    api.qmm_moe_gemv_id_gate_up_silu_batched(a.to(DEV).reshape(-1), ids.to(DEV), T, k, dm, 0,
                                             gate_s, up_s, out=gh16.out, d_status=status)
    api.qmm_moe_gemv_id(gh16.out.reshape(-1), ids.to(DEV).reshape(-1), T * k, dff, down_s,
                        out=go.out, d_status=status)
    torch.cuda.synchronize()
    h, h16, out = gh.check("gate_up"), gh16.check("gate_up bf16"), go.check("down")
    assert int(status.item()) == 0
    rne_equal(h16, h)
    a_np = np_storage(a).reshape(-1)
    ref_h, rc = oracle.moe_gate_up_silu_batched(a_np, oracle.BF16, ids.numpy(), T, k, dm, 0, og, ou)
    assert rc == oracle.ORC_OK
    gate(h.cpu().numpy(), ref_h, f"{case.name} gate_up_silu")
    h16_np = np_storage(h16).reshape(-1)
    ref_d, rc = oracle.moe_gemv_id(h16_np, oracle.BF16, ids.numpy().reshape(-1), T * k, dff, od)
    assert rc == oracle.ORC_OK
    gate(out.cpu().numpy(), ref_d, f"{case.name} down")


@pytest.mark.parametrize("gs,n_cols", [(64, 768), (32, 768), (128, 768), (64, 1280), (32, 256)])
@pytest.mark.parametrize("n_sel", [5, 24])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_moe_short_rows_one_copy_scales(gs, n_cols, n_sel, dtype):
    """Rows whose scale/bias rows are not 16-byte strided (K / gs = 12, 24, 6,
    20, 8 groups): the streaming kernel takes a whole row tile per unit and
    its 16 scale (bias) rows as one contiguous copy, skipping groups past the
    row; one pair per segment (5 pairs) and segments of 8 (24 pairs)."""
    E, n_rows, bits = 10, 96, 4
    st, ost = make_stack(E, n_rows, n_cols, bits, gs, 60 + gs + n_cols, dtype)
    stride = n_cols + 8
    dts = {torch.bfloat16: "bf16", torch.float16: "f16"}[dtype]
    a = wl.gen_x(1, stride * n_sel, 61, dts).reshape(-1)
    ids = torch.randint(0, E, (n_sel,), generator=torch.Generator().manual_seed(62), dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    g32, g16 = Guarded((n_sel, n_rows), torch.float32), Guarded((n_sel, n_rows), dtype)
    api.qmm_moe_gemv_id(a.to(DEV), ids.to(DEV), n_sel, stride, st, out=g32.out, d_status=status)
    api.qmm_moe_gemv_id(a.to(DEV), ids.to(DEV), n_sel, stride, st, out=g16.out, d_status=status)
    torch.cuda.synchronize()
    out32, out16 = g32.check("short rows"), g16.check("short rows 16-bit")
    assert int(status.item()) == 0
    ref, rc = oracle.moe_gemv_id(np_storage(a), ORC[dtype], ids.numpy(), n_sel, stride, ost)
    assert rc == oracle.ORC_OK
    gate(out32.cpu().numpy(), ref, f"short rows g{gs} K{n_cols} n{n_sel}")
    rne_equal(out16, out32)
