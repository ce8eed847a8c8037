"""Python binding of the C ABI (include/qmm.h), one function per entry point
with the same name.  Argument marshalling only: torch provides device memory
and the current stream; every step of the computation runs in libqmm.so.

Packed weights are held in torch.int32 tensors (the bit pattern of the
uint32 words).  All tensors must be CUDA tensors on the current device.
"""
from __future__ import annotations

import ctypes
import functools
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import (QMM_BF16, QMM_F16, QMM_F32, QMM_MODE_AFFINE, QMM_MODE_MXFP4, QMM_MODE_MXFP8,
                   QMM_MODE_NVFP4, QMM_U8, ExpertStackC, QWeightC, check)

_TO_CODE = {torch.float32: QMM_F32, torch.float16: QMM_F16, torch.bfloat16: QMM_BF16,
            torch.uint8: QMM_U8}
# bits and group size of the microscaled modes
MX_PARAMS = {QMM_MODE_MXFP4: (4, 32), QMM_MODE_MXFP8: (8, 32), QMM_MODE_NVFP4: (4, 16)}
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


def _need(t, what: str, numel: int, dtypes=None) -> None:
    """Refuse a tensor the kernels would read or write out of bounds: it must
    hold at least `numel` elements (of one of `dtypes` when given) and be
    contiguous.  Raises ValueError before any call into the library."""
    if t is None:
        raise ValueError(f"qmm: {what} is required")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"qmm: {what} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"qmm: {what} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"qmm: {what} holds {t.numel()} elements, the call needs {numel}")


def _on_device(**named) -> None:
    """Every given tensor is a CUDA tensor on the current device (where the
    library launches).  Raises ValueError otherwise."""
    cur = None
    for what, t in named.items():
        if t is None:
            continue
        d = t.get_device()  # -1: host memory
        if d < 0:
            raise ValueError(f"qmm: {what} must be a CUDA tensor, got one on {t.device}")
        if cur is None:
            cur = torch.cuda.current_device()
        if d != cur:
            raise ValueError(f"qmm: {what} is on {t.device}, but the current device is cuda:{cur} "
                             "(the call runs there)")


@functools.lru_cache(maxsize=1024)
def _words(cols: int, bits: int) -> int:
    wpr = qmm_packed_words_per_row(cols, bits)
    if wpr < 0:
        check("qmm", _lib.QMM_ERR_INVALID_ARG)
    return wpr


@functools.lru_cache(maxsize=1024)
def _groups(cols: int, group_size: int) -> int:
    G = qmm_groups_per_row(cols, group_size)
    if G < 0:
        check("qmm", _lib.QMM_ERR_INVALID_ARG)
    return G


_PACKED = (torch.int32,)
_FLOAT = (torch.float32, torch.float16, torch.bfloat16)


def _stream(stream=None) -> int:
    if stream is not None:
        return int(stream.cuda_stream)
    # the current stream's handle without building a Stream object
    return int(torch._C._cuda_getCurrentRawStream(torch.cuda.current_device()))


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

    def validate(self) -> dict:
        """packed, scales and biases hold rows x (words | groups) elements;
        returns them by name for the device check.  Microscaled modes: uint8
        scales, no biases."""
        n = self.rows
        if self.mode != QMM_MODE_AFFINE:
            if self.mode not in MX_PARAMS or MX_PARAMS[self.mode] != (self.bits, self.group_size):
                check("qmm", _lib.QMM_ERR_INVALID_ARG)
            if self.cols % self.group_size or self.cols % 32:
                check("qmm", _lib.QMM_ERR_INVALID_ARG)
            _need(self.packed, "packed", n * self.cols * self.bits // 32, _PACKED)
            _need(self.scales, "scales", n * (self.cols // self.group_size), (torch.uint8,))
            return {"packed": self.packed, "scales": self.scales}
        _need(self.packed, "packed", n * _words(self.cols, self.bits), _PACKED)
        G = _groups(self.cols, self.group_size)
        _need(self.scales, "scales", n * G, _FLOAT)
        _need(self.biases, "biases", n * G, (self.scales.dtype,))
        return {"packed": self.packed, "scales": self.scales, "biases": self.biases}

    def c(self) -> QWeightC:
        return QWeightC(_ptr(self.packed), _ptr(self.scales), _ptr(self.biases),
                        dtype_code(self.scales.dtype), self.rows, self.cols, self.group_size,
                        self.bits, self.mode)

    def prepared(self):
        """validate(), then (the CUDA device all the tensors are on, the C
        struct), or (None, None) when they are not all on one CUDA device.
        The result is kept while the fields and every tensor's data pointer,
        element count and dtype stay the same: a replaced, resized or retyped
        tensor is checked again before the next call."""
        p, s, b = self.packed, self.scales, self.biases
        key = (self.rows, self.cols, self.group_size, self.bits, self.mode,
               p.data_ptr(), p.numel(), p.dtype, s.data_ptr(), s.numel(), s.dtype,
               None if b is None else (b.data_ptr(), b.numel(), b.dtype))
        hit = self.__dict__.get("_prep")
        if hit is not None and hit[0] == key:
            return hit[1], hit[2]
        ws = self.validate()
        devs = {t.get_device() for t in ws.values()}
        if len(devs) != 1 or min(devs) < 0:
            return None, None
        dev, c = devs.pop(), self.c()
        self.__dict__["_prep"] = (key, dev, c)
        return dev, c


def mx_qweight(packed: torch.Tensor, scales: torch.Tensor, mode: int, rows: int, cols: int) -> QWeight:
    """A microscaled matrix (mxfp4 / mxfp8 / nvfp4): packed [rows,
    cols*bits/32] int32 lanes, scales [rows, cols/group_size] uint8 bytes."""
    bits, gs = MX_PARAMS[mode]
    return QWeight(packed, scales, None, rows, cols, gs, bits, mode)


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

    def validate(self, role: str = "") -> dict:
        """packed, scales and biases hold num_experts x n_rows x (words |
        groups) elements; returns them by name for the device check."""
        n = self.num_experts * self.n_rows
        _need(self.packed, role + "packed", n * _words(self.n_cols, self.bits), _PACKED)
        G = _groups(self.n_cols, self.group_size)
        _need(self.scales, role + "scales", n * G, _FLOAT)
        _need(self.biases, role + "biases", n * G, (self.scales.dtype,))
        return {role + "packed": self.packed, role + "scales": self.scales,
                role + "biases": self.biases}

    def c(self) -> ExpertStackC:
        return ExpertStackC(_ptr(self.packed), _ptr(self.scales), _ptr(self.biases),
                            dtype_code(self.scales.dtype), self.num_experts, self.n_rows,
                            self.n_cols, self.group_size, self.bits)

    def prepared(self, role: str = ""):
        """validate(role), then (the CUDA device all the tensors are on, the C
        struct), or (None, None) when they are not all on one CUDA device;
        kept like QWeight.prepared while nothing about the tensors changes."""
        p, s, b = self.packed, self.scales, self.biases
        key = (self.num_experts, self.n_rows, self.n_cols, self.group_size, self.bits,
               p.data_ptr(), p.numel(), p.dtype, s.data_ptr(), s.numel(), s.dtype,
               b.data_ptr(), b.numel(), b.dtype)
        hit = self.__dict__.get("_prep")
        if hit is not None and hit[0] == key:
            return hit[1], hit[2]
        ws = self.validate(role)
        devs = {t.get_device() for t in ws.values()}
        if len(devs) != 1 or min(devs) < 0:
            return None, None
        dev, c = devs.pop(), self.c()
        self.__dict__["_prep"] = (key, dev, c)
        return dev, c

    @staticmethod
    def from_qweight(q: "QWeight", num_experts: int) -> "ExpertStack":
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


def qmm_selftest_bounded_wait(spins: int, d_result: torch.Tensor, d_status: torch.Tensor,
                              stream=None) -> None:
    """Run the bounded-wait diagnostic kernel (see include/qmm.h)."""
    _need(d_result, "d_result", 3, (torch.int32,))
    _need(d_status, "d_status", 1, (torch.int32,))
    _on_device(d_result=d_result, d_status=d_status)
    rc = _lib.load().qmm_selftest_bounded_wait(int(spins), _ptr(d_result), _ptr(d_status),
                                               _stream(stream))
    check("qmm_selftest_bounded_wait", rc)


# ------------------------------------------------------------------ calls
def _last_pair_end(n_pairs: int, top_k: int, outer: int, inner: int, n_cols: int) -> int:
    """Elements of `a` the last pair reads up to (batched pair offsets)."""
    if n_pairs == 0:
        return 0
    last = n_pairs - 1
    return (last // top_k) * outer + (last % top_k) * inner + n_cols


def qmm_quantize(w: torch.Tensor, group_size: int = 64, bits: int = 4,
                 s_dtype: torch.dtype | None = None, stream=None) -> QWeight:
    """Dense [rows, cols] -> QWeight (scales/biases in s_dtype, default w.dtype)."""
    if w.dim() != 2:
        raise ValueError(f"qmm_quantize: w must be 2-D, got shape {tuple(w.shape)}")
    rows, cols = w.shape
    s_dtype = s_dtype or w.dtype
    wpr = qmm_packed_words_per_row(cols, bits)
    G = qmm_groups_per_row(cols, group_size)
    if wpr < 0 or G < 0:
        check("qmm_quantize", _lib.QMM_ERR_INVALID_ARG)
    w = w.contiguous()
    _need(w, "w", rows * cols, _FLOAT)
    _on_device(w=w)
    packed = torch.empty(rows, wpr, dtype=torch.int32, device=w.device)
    scales = torch.empty(rows, G, dtype=s_dtype, device=w.device)
    biases = torch.empty(rows, G, dtype=s_dtype, device=w.device)
    rc = _lib.load().qmm_quantize(_ptr(w), dtype_code(w.dtype), rows, cols, group_size, bits,
                                  dtype_code(s_dtype), _ptr(packed), _ptr(scales), _ptr(biases),
                                  _stream(stream))
    check("qmm_quantize", rc)
    return QWeight(packed, scales, biases, rows, cols, group_size, bits)


def qmm_dequantize(qw: QWeight, out_dtype: torch.dtype = torch.float32, out=None,
                   stream=None) -> torch.Tensor:
    ws = qw.validate()
    if out is None:
        out = torch.empty(qw.rows, qw.cols, dtype=out_dtype, device=qw.packed.device)
    _need(out, "out", qw.rows * qw.cols, _FLOAT)
    _on_device(out=out, **ws)
    c = qw.c()
    rc = _lib.load().qmm_dequantize(ctypes.byref(c), _ptr(out), dtype_code(out.dtype),
                                    _stream(stream))
    check("qmm_dequantize", rc)
    return out


def qmm_matmul(x: torch.Tensor, qw: QWeight, transpose: bool = True,
               y_dtype: torch.dtype | None = None, out=None, stream=None) -> torch.Tensor:
    """y = x . dequant(W)^T (transpose) or x . dequant(W); x [..., K]."""
    two_d = x.dim() == 2
    K = x.shape[-1]
    x2 = x if two_d and x.is_contiguous() else x.reshape(-1, K).contiguous()
    M = x2.shape[0]
    N = qw.rows if transpose else qw.cols
    _need(x2, "x", M * K, _FLOAT)
    wdev, c = qw.prepared()
    if out is None:
        out = torch.empty(M, N, dtype=y_dtype or x.dtype, device=x2.device)
    _need(out, "out", M * N, _FLOAT)
    if out.numel() != M * N:
        raise ValueError(f"qmm_matmul: out holds {out.numel()} elements, expected {M}x{N}")
    dx = x2.get_device()  # -1: host memory
    cur = torch.cuda.current_device() if dx >= 0 and c is not None else -1
    if not (dx == out.get_device() == wdev == cur):
        # the slow checks name the tensor that is elsewhere
        _on_device(x=x2, out=out)
        _on_device(**qw.validate())
        raise ValueError(f"qmm: the weights are not all on {x2.device}")
    st = int(stream.cuda_stream) if stream is not None else int(torch._C._cuda_getCurrentRawStream(cur))
    rc = _lib.load().qmm_matmul(x2.data_ptr(), dtype_code(x2.dtype), M, K, ctypes.byref(c),
                                int(bool(transpose)), out.data_ptr(), dtype_code(out.dtype), st)
    check("qmm_matmul", rc)
    return out if two_d and out.dim() == 2 and out.shape[0] == M else out.reshape(*x.shape[:-1], N)


def qmm_matmul_parts(x: torch.Tensor, parts, y_dtype: torch.dtype | None = None, out=None,
                     stream=None) -> torch.Tensor:
    """Fused projection: y[..., off_p : off_p + N_p] = x . dequant(W_p)^T for
    the QWeights in `parts` (same input dimension, any bits / group size /
    mode each); y is [..., sum N_p]."""
    parts = list(parts)
    if not parts:
        check("qmm_matmul_parts", _lib.QMM_ERR_INVALID_ARG)
    lead = x.shape[:-1]
    K = x.shape[-1]
    x2 = x.reshape(-1, K).contiguous()
    M = x2.shape[0]
    Ntot = sum(p.rows for p in parts)
    _need(x2, "x", M * K, _FLOAT)
    preps = []
    for i, p in enumerate(parts):
        try:
            preps.append(p.prepared())
        except ValueError as e:
            raise ValueError(f"qmm_matmul_parts: part {i}: {e}") from None
    if out is None:
        out = torch.empty(M, Ntot, dtype=y_dtype or x.dtype, device=x2.device)
    _need(out, "out", M * Ntot, _FLOAT)
    if out.numel() != M * Ntot:
        raise ValueError(f"qmm_matmul_parts: out holds {out.numel()} elements, expected {M}x{Ntot}")
    dx = x2.get_device()  # -1: host memory
    cur = torch.cuda.current_device() if dx >= 0 and all(c is not None for _, c in preps) else -1
    if not (dx == out.get_device() == cur and all(d == cur for d, _ in preps)):
        # the slow checks name the tensor that is elsewhere
        named = {}
        for i, p in enumerate(parts):
            named.update({f"part{i}.{k}": v for k, v in p.validate().items()})
        _on_device(x=x2, out=out, **named)
        raise ValueError(f"qmm_matmul_parts: the parts are not all on {x2.device}")
    arr = (QWeightC * len(parts))(*[c for _, c in preps])
    st = int(stream.cuda_stream) if stream is not None else int(torch._C._cuda_getCurrentRawStream(cur))
    rc = _lib.load().qmm_matmul_parts(x2.data_ptr(), dtype_code(x2.dtype), M, K, arr, len(parts),
                                      out.data_ptr(), dtype_code(out.dtype), st)
    check("qmm_matmul_parts", rc)
    return out.reshape(*lead, Ntot)


def qmm_quantize_dynamic_int8(w: torch.Tensor, stream=None):
    """Whole-tensor min/max int8: (q int8 with w's shape, params float32[4] on
    the device = {input_min, input_max, output_min, output_max})."""
    w = w.contiguous()
    _need(w, "w", w.numel(), _FLOAT)
    _on_device(w=w)
    q = torch.empty(w.shape, dtype=torch.int8, device=w.device)
    params = torch.empty(4, dtype=torch.float32, device=w.device)
    rc = _lib.load().qmm_quantize_dynamic_int8(_ptr(w), dtype_code(w.dtype), w.numel(), _ptr(q), _ptr(params),
                                               _stream(stream))
    check("qmm_quantize_dynamic_int8", rc)
    return q, params


def qmm_dequantize_dynamic_int8(q: torch.Tensor, params: torch.Tensor, out_dtype: torch.dtype = torch.float32,
                                out=None, stream=None) -> torch.Tensor:
    _need(q, "q", q.numel(), (torch.int8,))
    _need(params, "params", 4, (torch.float32,))
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    _need(out, "out", q.numel(), _FLOAT)
    _on_device(q=q, params=params, out=out)
    rc = _lib.load().qmm_dequantize_dynamic_int8(_ptr(q), q.numel(), _ptr(params), _ptr(out),
                                                 dtype_code(out.dtype), _stream(stream))
    check("qmm_dequantize_dynamic_int8", rc)
    return out


def qmm_matmul_dynamic_int8(x: torch.Tensor, q: torch.Tensor, params: torch.Tensor,
                            y_dtype: torch.dtype | None = None, out=None, stream=None) -> torch.Tensor:
    """y = x . w_hat^T for an int8 [N, K] weight with per-tensor params; x [..., K]."""
    if q.dim() != 2:
        raise ValueError(f"qmm_matmul_dynamic_int8: q must be 2-D [N, K], got {tuple(q.shape)}")
    N, K = q.shape
    lead = x.shape[:-1]
    if x.shape[-1] != K:
        check("qmm_matmul_dynamic_int8", _lib.QMM_ERR_INVALID_ARG)
    x2 = x.reshape(-1, K).contiguous()
    M = x2.shape[0]
    _need(x2, "x", M * K, _FLOAT)
    _need(q, "q", N * K, (torch.int8,))
    _need(params, "params", 4, (torch.float32,))
    if out is None:
        out = torch.empty(M, N, dtype=y_dtype or x.dtype, device=x2.device)
    _need(out, "out", M * N, _FLOAT)
    _on_device(x=x2, q=q, params=params, out=out)
    rc = _lib.load().qmm_matmul_dynamic_int8(_ptr(x2), dtype_code(x2.dtype), M, K, _ptr(q), N, _ptr(params),
                                             _ptr(out), dtype_code(out.dtype), _stream(stream))
    check("qmm_matmul_dynamic_int8", rc)
    return out.reshape(*lead, N)


def _moe_checks(a, ids, n_pairs, top_k, outer, inner, stacks, out, n_out_rows, d_status):
    """Sizes, dtypes and layouts, then one device for everything; returns the
    stacks' C structs."""
    _need(a, "a", _last_pair_end(n_pairs, top_k, outer, inner, stacks[0].n_cols), _FLOAT)
    preps = [st.prepared(role) for role, st in zip(("", "up."), stacks)]
    _need(ids, "ids", n_pairs, (torch.int32,))
    _need(out, "out", n_pairs * n_out_rows, _FLOAT)
    if d_status is not None:
        _need(d_status, "d_status", 1, (torch.int32,))
    da = a.get_device()  # -1: host memory
    cur = torch.cuda.current_device() if da >= 0 and all(c is not None for _, c in preps) else -1
    if not (da == cur and ids.get_device() == cur and out.get_device() == cur
            and (d_status is None or d_status.get_device() == cur) and all(d == cur for d, _ in preps)):
        # the slow checks name the tensor that is elsewhere
        named = {}
        for role, st in zip(("", "up."), stacks):
            named.update(st.validate(role))
        _on_device(a=a, ids=ids, out=out, d_status=d_status, **named)
        raise ValueError(f"qmm: the MoE arguments are not all on {a.device}")
    return [c for _, c in preps]


def qmm_moe_gemv_id(a: torch.Tensor, ids: torch.Tensor, n_selected: int, src1_stride: int,
                    w: ExpertStack, out_dtype: torch.dtype | None = None, out=None,
                    d_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(n_selected, w.n_rows, dtype=out_dtype or a.dtype, device=a.device)
    (c,) = _moe_checks(a, ids, n_selected, 1, src1_stride, 0, (w,), out, w.n_rows, d_status)
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
    if top_k > 0:
        (c,) = _moe_checks(a, ids, m * top_k, top_k, outer_stride, inner_stride, (w,), out, w.n_rows,
                           d_status)
    else:
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
    cg, cu = _moe_checks(a, ids, n_selected, 1, 0, 0, (gate, up), out, gate.n_rows, d_status)
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
    if top_k > 0:
        cg, cu = _moe_checks(a, ids, m * top_k, top_k, outer_stride, inner_stride, (gate, up), out,
                             gate.n_rows, d_status)
    else:
        cg, cu = gate.c(), up.c()
    rc = _lib.load().qmm_moe_gemv_id_gate_up_silu_batched(
        _ptr(a), dtype_code(a.dtype), _ptr(ids), m, top_k, outer_stride, inner_stride,
        ctypes.byref(cg), ctypes.byref(cu), _ptr(out), dtype_code(out.dtype), _ptr(d_status),
        _stream(stream))
    check("qmm_moe_gemv_id_gate_up_silu_batched", rc)
    return out


# ------------------------------------------------------------------ MoE prefill GEMM
def qmm_moe_gemm_workspace_bytes(n_pairs: int, num_experts: int) -> int:
    return int(_lib.load().qmm_moe_gemm_workspace_bytes(n_pairs, num_experts))


def qmm_moe_gemm_workspace_bytes_gathered(n_pairs: int, num_experts: int, n_cols: int) -> int:
    return int(_lib.load().qmm_moe_gemm_workspace_bytes_gathered(n_pairs, num_experts, n_cols))


def moe_workspace(n_pairs: int, num_experts: int, device=None, n_cols: int | None = None) -> torch.Tensor:
    """A device workspace of the size qmm_moe_compute_ids_tpe needs (int32);
    with n_cols, also room for the activation rows gathered in pair order
    (the GEMM then loads each tile's rows as one box)."""
    if n_cols is None:
        nb = qmm_moe_gemm_workspace_bytes(n_pairs, num_experts)
    else:
        nb = qmm_moe_gemm_workspace_bytes_gathered(n_pairs, num_experts, n_cols)
    if nb < 0:
        check("qmm_moe_gemm_workspace_bytes", _lib.QMM_ERR_INVALID_ARG)
    return torch.empty((nb + 3) // 4, dtype=torch.int32, device=device or "cuda")


def qmm_moe_compute_ids_tpe(ids: torch.Tensor, num_experts: int, workspace: torch.Tensor,
                            d_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Route the [batch, top_k] ids on the device into `workspace`."""
    n = ids.numel()
    _need(ids, "ids", n, (torch.int32,))
    _need(workspace, "workspace", 0, (torch.int32,))
    if d_status is not None:
        _need(d_status, "d_status", 1, (torch.int32,))
    _on_device(ids=ids, workspace=workspace, d_status=d_status)
    rc = _lib.load().qmm_moe_compute_ids_tpe(_ptr(ids), n, num_experts, _ptr(workspace),
                                             workspace.numel() * 4, _ptr(d_status), _stream(stream))
    check("qmm_moe_compute_ids_tpe", rc)
    return workspace


def qmm_moe_gemm_id(a: torch.Tensor, batch: int, top_k: int, ne11: int, workspace: torch.Tensor,
                    w: ExpertStack, out_dtype: torch.dtype | None = None, out=None,
                    stream=None) -> torch.Tensor:
    """out[p] = a[row(p)] . dequant(W[ids[p]])^T over the routed workspace;
    a is [batch * ne11, K] (ne11 = 1 or top_k); out is [batch * top_k, n_rows]."""
    n_pairs = batch * top_k
    if out is None:
        out = torch.empty(n_pairs, w.n_rows, dtype=out_dtype or a.dtype, device=a.device)
    _need(a, "a", batch * ne11 * w.n_cols, _FLOAT)
    named = w.validate()
    _need(workspace, "workspace", 0, (torch.int32,))
    _need(out, "out", n_pairs * w.n_rows, _FLOAT)
    _on_device(a=a, workspace=workspace, out=out, **named)
    c = w.c()
    rc = _lib.load().qmm_moe_gemm_id(_ptr(a), dtype_code(a.dtype), batch, top_k, ne11,
                                     _ptr(workspace), workspace.numel() * 4, ctypes.byref(c),
                                     _ptr(out), dtype_code(out.dtype), _stream(stream))
    check("qmm_moe_gemm_id", rc)
    return out


def qmm_moe_gemm_id_noalloc(a: torch.Tensor, ids: torch.Tensor, batch: int, top_k: int, ne11: int,
                            w: ExpertStack, out_dtype: torch.dtype | None = None, out=None,
                            d_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Routing and MoE prefill GEMM in one call, without a workspace: the
    schedule lives in the library's own fixed device scratch (at most 16384
    pairs and 256 experts; calls that overlap on the GPU race)."""
    n_pairs = batch * top_k
    if out is None:
        out = torch.empty(n_pairs, w.n_rows, dtype=out_dtype or a.dtype, device=a.device)
    _need(a, "a", batch * ne11 * w.n_cols, _FLOAT)
    named = w.validate()
    _need(ids, "ids", n_pairs, (torch.int32,))
    _need(out, "out", n_pairs * w.n_rows, _FLOAT)
    if d_status is not None:
        _need(d_status, "d_status", 1, (torch.int32,))
    _on_device(a=a, ids=ids, out=out, d_status=d_status, **named)
    c = w.c()
    rc = _lib.load().qmm_moe_gemm_id_noalloc(_ptr(a), dtype_code(a.dtype), _ptr(ids), batch, top_k, ne11,
                                             ctypes.byref(c), _ptr(out), dtype_code(out.dtype),
                                             _ptr(d_status), _stream(stream))
    check("qmm_moe_gemm_id_noalloc", rc)
    return out
