"""The C ABI without a GPU: the library loads, exports every function that
include/qmm.h declares, and rejects bad arguments on the host before any
CUDA call.  No computation is launched here."""
import ctypes
import os
import re

import pytest

from weight_only_quantized_qmm_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = open(os.path.join(ROOT, "include", "qmm.h")).read()


@pytest.fixture(scope="module")
def L():
    return _lib.load()


def declared_functions():
    body = re.sub(r"/\*.*?\*/", "", HEADER, flags=re.S)
    return sorted(set(re.findall(r"\b(qmm_[a-z0-9_]+)\s*\(", body)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert set(names) == set(_lib.EXPORTS), names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), f"{name} missing from libqmm.so"


def test_enum_values_match_header():
    for name, val in [("QMM_OK", 0), ("QMM_ERR_INVALID_ARG", 1), ("QMM_ERR_UNSUPPORTED", 2),
                      ("QMM_ERR_DTYPE", 3), ("QMM_ERR_ALIGNMENT", 4), ("QMM_ERR_CUDA", 5),
                      ("QMM_ERR_TIMEOUT", 6), ("QMM_ERR_BAD_EXPERT_ID", 7), ("QMM_F32", 0),
                      ("QMM_F16", 1), ("QMM_BF16", 2), ("QMM_U8", 3)]:
        assert re.search(rf"\b{name}\s*=\s*{val}\b", HEADER), name
        assert getattr(_lib, name) == val


def test_size_helpers(L):
    assert L.qmm_packed_words_per_row(4096, 4) == 512
    assert L.qmm_packed_words_per_row(4096, 3) == 384
    assert L.qmm_packed_words_per_row(32, 6) == 6
    assert L.qmm_packed_words_per_row(33, 3) == -1
    assert L.qmm_packed_words_per_row(64, 5) == -1
    assert L.qmm_groups_per_row(4096, 64) == 64
    assert L.qmm_groups_per_row(96, 64) == -1
    assert L.qmm_groups_per_row(64, 16) == -1
    for code in range(8):
        assert len(_lib.status_string(code)) > 0


A = 0x10000  # an aligned fake device address: never dereferenced by these calls


def qw(bits=4, gs=64, rows=8, cols=128, sdtype=_lib.QMM_BF16, mode=0, packed=A):
    return _lib.QWeightC(packed, A, A, sdtype, rows, cols, gs, bits, mode)


def matmul(L, w, x=A, x_dtype=_lib.QMM_BF16, M=1, K=128, transpose=1, y=A, y_dtype=_lib.QMM_BF16):
    return L.qmm_matmul(x, x_dtype, M, K, ctypes.byref(w), transpose, y, y_dtype, None)


def test_matmul_validation(L):
    assert matmul(L, qw(bits=5)) == _lib.QMM_ERR_INVALID_ARG
    assert matmul(L, qw(gs=48)) == _lib.QMM_ERR_INVALID_ARG
    assert matmul(L, qw(cols=96, gs=64)) == _lib.QMM_ERR_INVALID_ARG
    assert matmul(L, qw(mode=7)) == _lib.QMM_ERR_UNSUPPORTED
    # microscaled: scale bytes (QMM_U8), the mode's own bits and group size
    assert matmul(L, qw(mode=_lib.QMM_MODE_NVFP4)) == _lib.QMM_ERR_DTYPE
    assert matmul(L, qw(mode=_lib.QMM_MODE_NVFP4, sdtype=_lib.QMM_U8, bits=4, gs=32)) == _lib.QMM_ERR_INVALID_ARG
    assert matmul(L, qw(mode=_lib.QMM_MODE_MXFP8, sdtype=_lib.QMM_U8, bits=4, gs=32)) == _lib.QMM_ERR_INVALID_ARG
    assert matmul(L, qw(mode=_lib.QMM_MODE_MXFP4, sdtype=_lib.QMM_U8, bits=4, gs=32),
                  transpose=0) == _lib.QMM_ERR_UNSUPPORTED
    assert matmul(L, qw(), x_dtype=_lib.QMM_F16) == _lib.QMM_ERR_DTYPE
    assert matmul(L, qw(), y_dtype=_lib.QMM_F16) == _lib.QMM_ERR_DTYPE
    assert matmul(L, qw(), K=256) == _lib.QMM_ERR_INVALID_ARG
    assert matmul(L, qw(), transpose=2) == _lib.QMM_ERR_INVALID_ARG
    assert matmul(L, qw(packed=0)) == _lib.QMM_ERR_ALIGNMENT
    assert matmul(L, qw(packed=A + 4)) == _lib.QMM_ERR_ALIGNMENT
    assert matmul(L, qw(), x=A + 2) == _lib.QMM_ERR_ALIGNMENT
    assert matmul(L, qw(), M=-1) == _lib.QMM_ERR_INVALID_ARG
    assert matmul(L, qw(), M=0) == _lib.QMM_OK  # empty: nothing launched


def test_quantize_dequantize_validation(L):
    q = L.qmm_quantize
    assert q(A, 0, 4, 128, 64, 7, 2, A, A, A, None) == _lib.QMM_ERR_INVALID_ARG
    assert q(A, 0, 4, 100, 64, 4, 2, A, A, A, None) == _lib.QMM_ERR_INVALID_ARG
    assert q(A, 9, 4, 128, 64, 4, 2, A, A, A, None) == _lib.QMM_ERR_DTYPE
    assert q(A, 0, 4, 128, 64, 4, 2, A + 8, A, A, None) == _lib.QMM_ERR_ALIGNMENT
    assert q(A, 0, 0, 128, 64, 4, 2, A, A, A, None) == _lib.QMM_OK
    w = qw(rows=0)
    assert L.qmm_dequantize(ctypes.byref(w), A, _lib.QMM_F32, None) == _lib.QMM_OK
    w = qw(bits=1)
    assert L.qmm_dequantize(ctypes.byref(w), A, _lib.QMM_F32, None) == _lib.QMM_ERR_INVALID_ARG


def stack(E=4, rows=16, cols=128, bits=4, gs=64, sdtype=_lib.QMM_BF16):
    return _lib.ExpertStackC(A, A, A, sdtype, E, rows, cols, gs, bits)


def test_moe_validation(L):
    s = stack()
    f = L.qmm_moe_gemv_id
    assert f(A, _lib.QMM_BF16, A, 0, 128, ctypes.byref(s), A, _lib.QMM_BF16, None, None) == _lib.QMM_OK
    assert f(A, _lib.QMM_F16, A, 2, 128, ctypes.byref(s), A, _lib.QMM_F16, None, None) == _lib.QMM_ERR_DTYPE
    assert f(A, _lib.QMM_BF16, A + 2, 2, 128, ctypes.byref(s), A, _lib.QMM_BF16, None, None) == _lib.QMM_ERR_ALIGNMENT
    bad = stack(E=0)
    assert f(A, _lib.QMM_BF16, A, 2, 128, ctypes.byref(bad), A, _lib.QMM_BF16, None, None) == _lib.QMM_ERR_INVALID_ARG
    g, u = stack(), stack(rows=32)
    h = L.qmm_moe_gemv_id_gate_up_silu
    assert h(A, _lib.QMM_BF16, A, 2, ctypes.byref(g), ctypes.byref(u), A, _lib.QMM_BF16, None, None) == _lib.QMM_ERR_INVALID_ARG
    assert h(A, _lib.QMM_BF16, A, 2, ctypes.byref(g), None, A, _lib.QMM_BF16, None, None) == _lib.QMM_ERR_INVALID_ARG
    b = L.qmm_moe_gemv_id_batched
    assert b(A, _lib.QMM_BF16, A, 2, 0, 0, 0, ctypes.byref(s), A, _lib.QMM_BF16, None, None) == _lib.QMM_ERR_INVALID_ARG
    bb = L.qmm_moe_gemv_id_gate_up_silu_batched
    assert bb(A, _lib.QMM_BF16, A, 0, 8, 0, 0, ctypes.byref(g), ctypes.byref(g), A, _lib.QMM_BF16, None, None) == _lib.QMM_OK


def test_moe_limits_and_alignment(L):
    bf, f32 = _lib.QMM_BF16, _lib.QMM_F32
    s = stack()
    f = L.qmm_moe_gemv_id
    ok_args = dict(a=A, ids=A, out=A, status=None)

    def call(n=2, stride=128, w=s, a_dtype=bf, out_dtype=bf, **kw):
        args = {**ok_args, **kw}
        return f(args["a"], a_dtype, args["ids"], n, stride, ctypes.byref(w), args["out"],
                 out_dtype, args["status"], None)

    # dtype rules: out is a_dtype or f32; fp32 activations have no MoE kernel
    assert call(out_dtype=_lib.QMM_F16) == _lib.QMM_ERR_DTYPE
    s32 = stack(sdtype=f32)
    assert call(w=s32, a_dtype=f32, out_dtype=f32) == _lib.QMM_ERR_UNSUPPORTED
    # negative counts and strides
    assert call(n=-1) == _lib.QMM_ERR_INVALID_ARG
    assert call(stride=-128) == _lib.QMM_ERR_INVALID_ARG
    # size limits: 65536 pairs and 65536 experts
    assert call(n=65537) == _lib.QMM_ERR_UNSUPPORTED
    assert call(w=stack(E=65537)) == _lib.QMM_ERR_UNSUPPORTED
    # pointer rules: a needs element alignment, ids and d_status 4 bytes, out 16
    assert call(a=0) == _lib.QMM_ERR_ALIGNMENT
    assert call(a=A + 1) == _lib.QMM_ERR_ALIGNMENT
    assert call(ids=A + 2) == _lib.QMM_ERR_ALIGNMENT
    assert call(ids=0) == _lib.QMM_ERR_ALIGNMENT
    assert call(status=A + 2) == _lib.QMM_ERR_ALIGNMENT
    assert call(out=A + 8) == _lib.QMM_ERR_ALIGNMENT


def test_moe_batched_pair_count_cannot_overflow(L):
    """m * top_k is checked against the 65536-pair limit without forming a
    product that wraps (2^32 * 2^32 would wrap to 0 pairs)."""
    s = stack()
    g = stack()
    b = L.qmm_moe_gemv_id_batched
    bb = L.qmm_moe_gemv_id_gate_up_silu_batched
    bf = _lib.QMM_BF16
    for m, top_k, want in [(2**32, 2**32, _lib.QMM_ERR_UNSUPPORTED),
                           (2**62, 4, _lib.QMM_ERR_UNSUPPORTED),
                           (1000, 66, _lib.QMM_ERR_UNSUPPORTED),
                           (0, 2**40, _lib.QMM_OK),
                           (-1, 8, _lib.QMM_ERR_INVALID_ARG),
                           (4, 0, _lib.QMM_ERR_INVALID_ARG)]:
        assert b(A, bf, A, m, top_k, 0, 0, ctypes.byref(s), A, bf, None, None) == want, (m, top_k)
        assert bb(A, bf, A, m, top_k, 0, 0, ctypes.byref(g), ctypes.byref(g), A, bf, None,
                  None) == want, (m, top_k)
    assert b(A, bf, A, 2, 4, -1, 0, ctypes.byref(s), A, bf, None, None) == _lib.QMM_ERR_INVALID_ARG
    assert b(A, bf, A, 2, 4, 0, -1, ctypes.byref(s), A, bf, None, None) == _lib.QMM_ERR_INVALID_ARG


def test_moe_gate_up_must_match(L):
    h = L.qmm_moe_gemv_id_gate_up_silu
    bf = _lib.QMM_BF16
    g = stack()
    for up in (stack(E=5), stack(cols=256), stack(bits=8), stack(gs=32),
               stack(sdtype=_lib.QMM_F16)):
        assert h(A, bf, A, 2, ctypes.byref(g), ctypes.byref(up), A, bf, None, None) \
            == _lib.QMM_ERR_INVALID_ARG


def _sources(root, exts):
    for dirpath, dirnames, files in os.walk(root):
        dirnames[:] = [d for d in dirnames if not d.startswith((".", "_build", "__pycache__"))]
        for f in files:
            if f.endswith(exts):
                yield os.path.join(dirpath, f)


def test_product_and_oracle_share_no_code():
    """The product package never loads the oracle, and the oracle never
    includes, imports or links anything of the product."""
    pkg = os.path.join(ROOT, "weight_only_quantized_qmm_b200")
    bad_in_pkg = re.compile(r"^\s*(import|from)\s+oracle\b|liboracle|qmm_oracle\.c", re.M)
    for path in _sources(pkg, (".py", ".cu", ".cuh", ".h", ".cpp")):
        assert not bad_in_pkg.search(open(path).read()), path
    bad_in_oracle = re.compile(r"weight_only_quantized_qmm_b200|libqmm|#include\s+\"|qmm\.h")
    for path in _sources(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        assert not bad_in_oracle.search(open(path).read()), path


def test_binding_refuses_host_tensors():
    """The Python binding passes device addresses only: a CPU tensor raises
    before anything reaches the library (no CPU path exists)."""
    import torch

    from weight_only_quantized_qmm_b200 import api

    with pytest.raises(ValueError, match="CUDA"):
        api.qmm_quantize(torch.zeros(16, 64), 32, 4)
    qw = api.QWeight(torch.zeros(16, 8, dtype=torch.int32), torch.zeros(16, 2),
                     torch.zeros(16, 2), 16, 64, 32, 4)
    with pytest.raises(ValueError, match="CUDA"):
        api.qmm_matmul(torch.zeros(1, 64), qw)
    with pytest.raises(ValueError, match="CUDA"):
        api.qmm_dequantize(qw)


def test_parts_validation(L):
    arr = (_lib.QWeightC * 2)(qw(), qw(rows=16))
    call = lambda parts, n, K=128, x_dtype=_lib.QMM_BF16, M=1, y=A: L.qmm_matmul_parts(  # noqa: E731
        A, x_dtype, M, K, parts, n, y, _lib.QMM_BF16, None)
    assert call(None, 2) == _lib.QMM_ERR_INVALID_ARG
    assert call(arr, 0) == _lib.QMM_ERR_INVALID_ARG
    assert call(arr, 65) == _lib.QMM_ERR_INVALID_ARG
    assert call(arr, 2, K=256) == _lib.QMM_ERR_INVALID_ARG      # a part's input dimension differs
    assert call(arr, 2, x_dtype=_lib.QMM_F16) == _lib.QMM_ERR_DTYPE
    bad = (_lib.QWeightC * 2)(qw(), qw(bits=5))
    assert call(bad, 2) == _lib.QMM_ERR_INVALID_ARG             # every part is checked first
    assert call(arr, 2, M=0) == _lib.QMM_OK                     # nothing to do
    assert call(arr, 2, y=A + 8) == _lib.QMM_ERR_ALIGNMENT


def test_dynamic_int8_validation(L):
    q = L.qmm_quantize_dynamic_int8
    assert q(A, 9, 16, A, A, None) == _lib.QMM_ERR_DTYPE
    assert q(A, _lib.QMM_F32, 0, A, A, None) == _lib.QMM_ERR_INVALID_ARG
    assert q(A, _lib.QMM_F32, 16, A + 4, A, None) == _lib.QMM_ERR_ALIGNMENT
    assert q(A, _lib.QMM_F32, 16, A, A + 2, None) == _lib.QMM_ERR_ALIGNMENT
    d = L.qmm_dequantize_dynamic_int8
    assert d(A, -1, A, A, _lib.QMM_F32, None) == _lib.QMM_ERR_INVALID_ARG
    assert d(A, 0, A, A, _lib.QMM_F32, None) == _lib.QMM_OK
    assert d(A, 16, A, A, 9, None) == _lib.QMM_ERR_DTYPE
    assert d(A, 16, None, A, _lib.QMM_F32, None) == _lib.QMM_ERR_ALIGNMENT
    m = L.qmm_matmul_dynamic_int8
    assert m(A, _lib.QMM_BF16, 1, 64, A, 8, A, A, _lib.QMM_F16, None) == _lib.QMM_ERR_DTYPE
    assert m(A, _lib.QMM_BF16, -1, 64, A, 8, A, A, _lib.QMM_BF16, None) == _lib.QMM_ERR_INVALID_ARG
    assert m(A, _lib.QMM_BF16, 1, 0, A, 8, A, A, _lib.QMM_BF16, None) == _lib.QMM_ERR_INVALID_ARG
    assert m(A, _lib.QMM_BF16, 0, 64, A, 8, A, A, _lib.QMM_BF16, None) == _lib.QMM_OK
    assert m(A, _lib.QMM_BF16, 1, 64, A + 1, 8, A, A, _lib.QMM_BF16, None) == _lib.QMM_ERR_ALIGNMENT
