"""Python binding of the C ABI (include/qmm.h), one function per entry point
with the same name.  Argument marshalling only: torch provides device memory
and the current stream; every step of the computation runs in libqmm.so.

Packed weights are held in torch.int32 tensors (the bit pattern of the
uint32 words).  All tensors must be CUDA tensors on the current device.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import QMM_BF16, QMM_F16, QMM_F32, QMM_MODE_AFFINE, ExpertStackC, QWeightC, check

_TO_CODE = {torch.float32: QMM_F32, torch.float16: QMM_F16, torch.bfloat16: QMM_BF16}
_FROM_CODE = {v: k for k, v in _TO_CODE.items()}


def dtype_code(dt: torch.dtype) -> int:
    try:
        return _TO_CODE[dt]
    except KeyError:
        raise TypeError(f"unsupported dtype {dt}") from None


def _ptr(t) -> int:
    """Device address of a CUDA tensor (0 for None).  A host tensor is
    refused: the kernels would dereference its address on the GPU."""
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"qmm: tensor arguments must be CUDA tensors, got one on {t.device}")
    return int(t.data_ptr())


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


@dataclass
class QWeight:
    """A quantized matrix: packed [rows, cols*bits/32] int32 (uint32 bits),
    scales/biases [rows, cols/group_size]; the quantized axis is `cols`."""
    packed: torch.Tensor
    scales: torch.Tensor
    biases: torch.Tensor
    rows: int
    cols: int
    group_size: int
    bits: int
    mode: int = QMM_MODE_AFFINE

    def c(self) -> QWeightC:
        return QWeightC(_ptr(self.packed), _ptr(self.scales), _ptr(self.biases),
                        dtype_code(self.scales.dtype), self.rows, self.cols, self.group_size,
                        self.bits, self.mode)


@dataclass
class ExpertStack:
    """num_experts matrices [n_rows, n_cols] of one role stored contiguously."""
    packed: torch.Tensor
    scales: torch.Tensor
    biases: torch.Tensor
    num_experts: int
    n_rows: int
    n_cols: int
    group_size: int
    bits: int

    def c(self) -> ExpertStackC:
        return ExpertStackC(_ptr(self.packed), _ptr(self.scales), _ptr(self.biases),
                            dtype_code(self.scales.dtype), self.num_experts, self.n_rows,
                            self.n_cols, self.group_size, self.bits)

    @staticmethod
    def from_qweight(q: QWeight, num_experts: int) -> "ExpertStack":
        assert q.rows % num_experts == 0
        return ExpertStack(q.packed, q.scales, q.biases, num_experts, q.rows // num_experts,
                           q.cols, q.group_size, q.bits)


# ------------------------------------------------------------------ helpers
def qmm_packed_words_per_row(cols: int, bits: int) -> int:
    return int(_lib.load().qmm_packed_words_per_row(cols, bits))


def qmm_groups_per_row(cols: int, group_size: int) -> int:
    return int(_lib.load().qmm_groups_per_row(cols, group_size))


def qmm_status_string(code: int) -> str:
    return _lib.status_string(code)


def qmm_device_check() -> int:
    return int(_lib.load().qmm_device_check())


# ------------------------------------------------------------------ calls
def qmm_quantize(w: torch.Tensor, group_size: int = 64, bits: int = 4,
                 s_dtype: torch.dtype | None = None, stream=None) -> QWeight:
    """Dense [rows, cols] -> QWeight (scales/biases in s_dtype, default w.dtype)."""
    rows, cols = w.shape
    s_dtype = s_dtype or w.dtype
    wpr = qmm_packed_words_per_row(cols, bits)
    G = qmm_groups_per_row(cols, group_size)
    if wpr < 0 or G < 0:
        check("qmm_quantize", _lib.QMM_ERR_INVALID_ARG)
    packed = torch.empty(rows, wpr, dtype=torch.int32, device=w.device)
    scales = torch.empty(rows, G, dtype=s_dtype, device=w.device)
    biases = torch.empty(rows, G, dtype=s_dtype, device=w.device)
    w = w.contiguous()
    rc = _lib.load().qmm_quantize(_ptr(w), dtype_code(w.dtype), rows, cols, group_size, bits,
                                  dtype_code(s_dtype), _ptr(packed), _ptr(scales), _ptr(biases),
                                  _stream(stream))
    check("qmm_quantize", rc)
    return QWeight(packed, scales, biases, rows, cols, group_size, bits)


def qmm_dequantize(qw: QWeight, out_dtype: torch.dtype = torch.float32, out=None,
                   stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(qw.rows, qw.cols, dtype=out_dtype, device=qw.packed.device)
    c = qw.c()
    rc = _lib.load().qmm_dequantize(ctypes.byref(c), _ptr(out), dtype_code(out.dtype),
                                    _stream(stream))
    check("qmm_dequantize", rc)
    return out


def qmm_matmul(x: torch.Tensor, qw: QWeight, transpose: bool = True,
               y_dtype: torch.dtype | None = None, out=None, stream=None) -> torch.Tensor:
    """y = x . dequant(W)^T (transpose) or x . dequant(W); x [..., K]."""
    lead = x.shape[:-1]
    K = x.shape[-1]
    x2 = x.reshape(-1, K).contiguous()
    M = x2.shape[0]
    N = qw.rows if transpose else qw.cols
    if out is None:
        out = torch.empty(M, N, dtype=y_dtype or x.dtype, device=x.device)
    c = qw.c()
    rc = _lib.load().qmm_matmul(_ptr(x2), dtype_code(x2.dtype), M, K, ctypes.byref(c),
                                int(bool(transpose)), _ptr(out), dtype_code(out.dtype),
                                _stream(stream))
    check("qmm_matmul", rc)
    return out.reshape(*lead, N)


def qmm_moe_gemv_id(a: torch.Tensor, ids: torch.Tensor, n_selected: int, src1_stride: int,
                    w: ExpertStack, out_dtype: torch.dtype | None = None, out=None,
                    d_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(n_selected, w.n_rows, dtype=out_dtype or a.dtype, device=a.device)
    c = w.c()
    rc = _lib.load().qmm_moe_gemv_id(_ptr(a), dtype_code(a.dtype), _ptr(ids), n_selected,
                                     src1_stride, ctypes.byref(c), _ptr(out),
                                     dtype_code(out.dtype), _ptr(d_status), _stream(stream))
    check("qmm_moe_gemv_id", rc)
    return out


def qmm_moe_gemv_id_batched(a: torch.Tensor, ids: torch.Tensor, m: int, top_k: int,
                            outer_stride: int, inner_stride: int, w: ExpertStack,
                            out_dtype: torch.dtype | None = None, out=None,
                            d_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(m * top_k, w.n_rows, dtype=out_dtype or a.dtype, device=a.device)
    c = w.c()
    rc = _lib.load().qmm_moe_gemv_id_batched(_ptr(a), dtype_code(a.dtype), _ptr(ids), m, top_k,
                                             outer_stride, inner_stride, ctypes.byref(c),
                                             _ptr(out), dtype_code(out.dtype), _ptr(d_status),
                                             _stream(stream))
    check("qmm_moe_gemv_id_batched", rc)
    return out


def qmm_moe_gemv_id_gate_up_silu(a: torch.Tensor, ids: torch.Tensor, n_selected: int,
                                 gate: ExpertStack, up: ExpertStack,
                                 out_dtype: torch.dtype | None = None, out=None,
                                 d_status: torch.Tensor | None = None,
                                 stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(n_selected, gate.n_rows, dtype=out_dtype or a.dtype, device=a.device)
    cg, cu = gate.c(), up.c()
    rc = _lib.load().qmm_moe_gemv_id_gate_up_silu(_ptr(a), dtype_code(a.dtype), _ptr(ids),
                                                  n_selected, ctypes.byref(cg), ctypes.byref(cu),
                                                  _ptr(out), dtype_code(out.dtype),
                                                  _ptr(d_status), _stream(stream))
    check("qmm_moe_gemv_id_gate_up_silu", rc)
    return out


def qmm_moe_gemv_id_gate_up_silu_batched(a: torch.Tensor, ids: torch.Tensor, m: int, top_k: int,
                                         outer_stride: int, inner_stride: int,
                                         gate: ExpertStack, up: ExpertStack,
                                         out_dtype: torch.dtype | None = None, out=None,
                                         d_status: torch.Tensor | None = None,
                                         stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(m * top_k, gate.n_rows, dtype=out_dtype or a.dtype, device=a.device)
    cg, cu = gate.c(), up.c()
    rc = _lib.load().qmm_moe_gemv_id_gate_up_silu_batched(
        _ptr(a), dtype_code(a.dtype), _ptr(ids), m, top_k, outer_stride, inner_stride,
        ctypes.byref(cg), ctypes.byref(cu), _ptr(out), dtype_code(out.dtype), _ptr(d_status),
        _stream(stream))
    check("qmm_moe_gemv_id_gate_up_silu_batched", rc)
    return out
