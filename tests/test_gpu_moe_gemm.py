"""GPU parity of the MoE prefill path: the on-device routing
(qmm_moe_compute_ids_tpe: tokens per expert, pairs grouped by expert, work
blocks, the 12-byte triple) and the expert-grouped tcgen05 GEMM
(qmm_moe_gemm_id), through the C ABI, against the CPU oracle."""
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
    return api.ExpertStack.from_qweight(qw, E), oracle.Stack(p, s, b, ORC[dtype], E, n_rows, n_cols, gs, bits)


def ws_fields(ws, n_pairs, E):
    """the workspace fields, at the offsets include/qmm.h documents"""
    v = ws.cpu().numpy()
    r4 = lambda n: (n + 3) // 4 * 4  # noqa: E731
    nb = (n_pairs + 255) // 256 + E
    o_pairs = r4(2 * E + 4)
    o_be = o_pairs + r4(n_pairs)
    o_bs = o_be + r4(nb)
    return dict(tpe=v[:E], off=v[E:2 * E + 1], args=v[2 * E + 1:2 * E + 4],
                pairs=v[o_pairs:o_pairs + n_pairs], blk_e=v[o_be:o_be + nb], blk_s=v[o_bs:o_bs + nb])


@pytest.mark.parametrize("batch,top_k,E", [(1, 1, 4), (37, 4, 16), (300, 8, 128), (64, 2, 3)])
def test_routing_workspace(batch, top_k, E):
    ids = wl.gen_moe_ids(batch, E, top_k, 70 + batch) if top_k <= E else None
    P = batch * top_k
    ws = api.moe_workspace(P, E)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    api.qmm_moe_compute_ids_tpe(ids.to(DEV), E, ws, status)
    torch.cuda.synchronize()
    f = ws_fields(ws, P, E)
    flat = ids.numpy().reshape(-1)
    cnt = np.bincount(flat, minlength=E)
    assert np.array_equal(f["tpe"], cnt)
    assert np.array_equal(f["off"], np.concatenate([[0], np.cumsum(cnt)]))
    nblk = int(sum((c + 255) // 256 for c in cnt))
    assert list(f["args"]) == [nblk, int(cnt.max()), int((cnt > 0).sum())]
    for e in range(E):  # every expert's group holds exactly its pairs
        grp = f["pairs"][f["off"][e]:f["off"][e + 1]]
        assert np.array_equal(np.sort(grp), np.nonzero(flat == e)[0])
    # blocks tile every group in order, <= 256 pairs each
    blocks = [(int(f["blk_e"][b]), int(f["blk_s"][b])) for b in range(nblk)]
    exp = [(e, int(f["off"][e]) + 256 * k) for e in range(E) for k in range((cnt[e] + 255) // 256)]
    assert blocks == exp
    assert int(status.item()) == 0


def _moe_gemm_case(batch, top_k, ne11, E, n_rows, n_cols, bits, gs, dtype, seed, bad=(), gathered=False):
    st, ost = make_stack(E, n_rows, n_cols, bits, gs, seed, dtype)
    ids = wl.gen_moe_ids(batch, E, top_k, seed + 1)
    for (t, k) in bad:
        ids[t, k] = E + 5 if (t + k) % 2 else -1
    P = batch * top_k
    dts = {torch.bfloat16: "bf16", torch.float16: "f16"}[dtype]
    a = wl.gen_x(batch * ne11, n_cols, seed + 2, dts)
    ws = api.moe_workspace(P, E, n_cols=n_cols if gathered else None)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    g32, g16 = Guarded((P, n_rows), torch.float32), Guarded((P, n_rows), dtype)
    api.qmm_moe_compute_ids_tpe(ids.to(DEV), E, ws, status)
    api.qmm_moe_gemm_id(a.to(DEV), batch, top_k, ne11, ws, st, out=g32.out)
    api.qmm_moe_gemm_id(a.to(DEV), batch, top_k, ne11, ws, st, out=g16.out)
    torch.cuda.synchronize()
    out32, out16 = g32.check("moe gemm"), g16.check("moe gemm 16-bit")
    outer, inner = (n_cols, 0) if ne11 == 1 else (top_k * n_cols, n_cols)
    ref, rc = oracle.moe_batched_dense(np_storage(a), ORC[dtype], ids.numpy(), batch, top_k, outer, inner, ost)
    return out32, out16, ref, rc, int(status.item()), ids


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 32), (3, 128), (2, 64), (6, 64)])
@pytest.mark.parametrize("ne11", [1, 4])
@pytest.mark.parametrize("gathered", [False, True])
def test_moe_gemm_widths_and_layouts(bits, gs, ne11, gathered):
    out32, out16, ref, rc, st, _ = _moe_gemm_case(70, 4, ne11, 12, 200, 256, bits, gs, torch.bfloat16,
                                                  800 + bits + gs + ne11, gathered=gathered)
    assert rc == oracle.ORC_OK and st == 0
    gate(out32.cpu().numpy(), ref, f"moe gemm b{bits} g{gs} ne11={ne11}")
    rne_equal(out16, out32)


@pytest.mark.parametrize("E", [128, 40])
def test_moe_gemm_gathered_rows_give_the_same_bits(E):
    """the workspace with room for the gathered rows changes how the rows
    reach the tile, not the arithmetic: both paths agree bit for bit (E = 128:
    ~19 pairs per expert; E = 40: ~60)"""
    a32, a16, *_ = _moe_gemm_case(300, 8, 1, E, 256, 512, 4, 64, torch.bfloat16, 880)
    b32, b16, *_ = _moe_gemm_case(300, 8, 1, E, 256, 512, 4, 64, torch.bfloat16, 880, gathered=True)
    assert torch.equal(a32.view(torch.int32), b32.view(torch.int32))
    assert torch.equal(a16.view(torch.int16), b16.view(torch.int16))


@pytest.mark.parametrize("gathered", [False, True])
def test_moe_gemm_fp16_and_many_blocks_per_expert(gathered):
    """an expert with more than 256 pairs spans several blocks"""
    out32, out16, ref, rc, st, ids = _moe_gemm_case(700, 2, 1, 3, 160, 512, 4, 64, torch.float16, 850,
                                                    gathered=gathered)
    assert int(np.bincount(ids.numpy().reshape(-1)).max()) > 256
    gate(out32.cpu().numpy(), ref, "moe gemm f16 long groups")
    rne_equal(out16, out32)


def test_moe_gemm_bad_ids_zero_rows_and_status():
    bad = [(3, 1), (10, 0), (11, 3)]
    out32, _, ref, rc, st, ids = _moe_gemm_case(40, 4, 4, 8, 128, 256, 4, 64, torch.bfloat16, 870, bad, gathered=True)
    assert rc == oracle.ORC_ERR_ID and st & 7 == 7
    o = out32.cpu().numpy()
    for (t, k) in bad:
        assert np.all(o[t * 4 + k] == 0)
    gate(o, ref, "moe gemm with bad ids")


@pytest.mark.parametrize("T", [256, 2048])
def test_moe_prefill_full_size(T):
    """128 experts, top-8: gate and up [768 x 2048] read the token rows
    (ne11 = 1), down [2048 x 768] reads one row per pair (ne11 = 8); every
    output of the three GEMMs against the oracle."""
    E, dff, dm, k = 128, 768, 2048, 8
    gate_s, og = make_stack(E, dff, dm, 4, 64, 4500 + T)
    down_s, od = make_stack(E, dm, dff, 4, 64, 4501 + T)
    ids = wl.gen_moe_ids(T, E, k, 4502 + T)
    a = wl.gen_x(T, dm, 4503 + T)
    P = T * k
    ws = api.moe_workspace(P, E, n_cols=dm)  # room for the gathered rows of either projection
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gg = Guarded((P, dff), torch.float32)
    api.qmm_moe_compute_ids_tpe(ids.to(DEV), E, ws, status)
    api.qmm_moe_gemm_id(a.to(DEV), T, k, 1, ws, gate_s, out=gg.out)
    h = wl.gen_x(P, dff, 4504 + T)  # per-pair activations of the down projection
    gd = Guarded((P, dm), torch.float32)
    api.qmm_moe_gemm_id(h.to(DEV), T, k, k, ws, down_s, out=gd.out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, rc = oracle.moe_batched_dense(np_storage(a), oracle.BF16, ids.numpy(), T, k, dm, 0, og)
    gate(gg.check("gate").cpu().numpy(), ref, f"moe prefill T{T} gate")
    ref, rc = oracle.moe_batched_dense(np_storage(h), oracle.BF16, ids.numpy(), T, k, k * dff, dff, od)
    gate(gd.check("down").cpu().numpy(), ref, f"moe prefill T{T} down")
