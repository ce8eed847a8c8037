"""ctypes loader for libqmm.so (the C ABI declared in include/qmm.h).

The library is built in-tree (``python -m weight_only_quantized_qmm_b200.build``
or ``__graft_entry__.build()``).  There is no fallback: a missing library is
an ImportError-style failure raised at first use.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libqmm.so")

QMM_OK = 0
QMM_ERR_INVALID_ARG = 1
QMM_ERR_UNSUPPORTED = 2
QMM_ERR_DTYPE = 3
QMM_ERR_ALIGNMENT = 4
QMM_ERR_CUDA = 5
QMM_ERR_TIMEOUT = 6
QMM_ERR_BAD_EXPERT_ID = 7

QMM_F32, QMM_F16, QMM_BF16, QMM_U8 = 0, 1, 2, 3
QMM_MODE_AFFINE, QMM_MODE_MXFP4, QMM_MODE_MXFP8, QMM_MODE_NVFP4 = 0, 1, 2, 3

# every symbol include/qmm.h declares
EXPORTS = (
    "qmm_packed_words_per_row", "qmm_groups_per_row", "qmm_status_string", "qmm_device_check",
    "qmm_quantize", "qmm_dequantize", "qmm_matmul", "qmm_moe_gemv_id",
    "qmm_moe_gemv_id_batched", "qmm_moe_gemv_id_gate_up_silu",
    "qmm_moe_gemv_id_gate_up_silu_batched", "qmm_moe_gemm_workspace_bytes",
    "qmm_moe_compute_ids_tpe", "qmm_moe_gemm_id", "qmm_moe_gemm_id_noalloc",
    "qmm_selftest_bounded_wait", "qmm_matmul_parts", "qmm_quantize_dynamic_int8",
    "qmm_dequantize_dynamic_int8", "qmm_matmul_dynamic_int8", "qmm_moe_gemm_workspace_bytes_gathered",
)


class QWeightC(ctypes.Structure):
    """qmm_qweight"""
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p), ("sdtype", ctypes.c_int),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("group_size", ctypes.c_int), ("bits", ctypes.c_int), ("mode", ctypes.c_int)]


class ExpertStackC(ctypes.Structure):
    """qmm_expert_stack"""
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p), ("sdtype", ctypes.c_int),
                ("num_experts", ctypes.c_int64), ("n_rows", ctypes.c_int64),
                ("n_cols", ctypes.c_int64), ("group_size", ctypes.c_int), ("bits", ctypes.c_int)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libqmm.so once; raise a clear error when it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libqmm.so not found at {LIB_PATH}: build it with "
            "`python -m weight_only_quantized_qmm_b200.build` (there is no fallback path)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    qwp = ctypes.POINTER(QWeightC)
    stp = ctypes.POINTER(ExpertStackC)
    L.qmm_packed_words_per_row.argtypes = [i64, c_int]
    L.qmm_packed_words_per_row.restype = i64
    L.qmm_groups_per_row.argtypes = [i64, c_int]
    L.qmm_groups_per_row.restype = i64
    L.qmm_status_string.argtypes = [c_int]
    L.qmm_status_string.restype = ctypes.c_char_p
    L.qmm_device_check.argtypes = []
    L.qmm_device_check.restype = c_int
    L.qmm_quantize.argtypes = [vp, c_int, i64, i64, c_int, c_int, c_int, vp, vp, vp, vp]
    L.qmm_quantize.restype = c_int
    L.qmm_dequantize.argtypes = [qwp, vp, c_int, vp]
    L.qmm_dequantize.restype = c_int
    L.qmm_matmul.argtypes = [vp, c_int, i64, i64, qwp, c_int, vp, c_int, vp]
    L.qmm_matmul.restype = c_int
    L.qmm_moe_gemv_id.argtypes = [vp, c_int, vp, i64, i64, stp, vp, c_int, vp, vp]
    L.qmm_moe_gemv_id.restype = c_int
    L.qmm_moe_gemv_id_batched.argtypes = [vp, c_int, vp, i64, i64, i64, i64, stp, vp, c_int, vp,
                                          vp]
    L.qmm_moe_gemv_id_batched.restype = c_int
    L.qmm_moe_gemv_id_gate_up_silu.argtypes = [vp, c_int, vp, i64, stp, stp, vp, c_int, vp, vp]
    L.qmm_moe_gemv_id_gate_up_silu.restype = c_int
    L.qmm_moe_gemv_id_gate_up_silu_batched.argtypes = [vp, c_int, vp, i64, i64, i64, i64, stp,
                                                       stp, vp, c_int, vp, vp]
    L.qmm_moe_gemv_id_gate_up_silu_batched.restype = c_int
    L.qmm_moe_gemm_workspace_bytes.argtypes = [i64, i64]
    L.qmm_moe_gemm_workspace_bytes.restype = i64
    L.qmm_moe_gemm_workspace_bytes_gathered.argtypes = [i64, i64, i64]
    L.qmm_moe_gemm_workspace_bytes_gathered.restype = i64
    L.qmm_moe_compute_ids_tpe.argtypes = [vp, i64, i64, vp, i64, vp, vp]
    L.qmm_moe_compute_ids_tpe.restype = c_int
    L.qmm_moe_gemm_id.argtypes = [vp, c_int, i64, i64, i64, vp, i64, stp, vp, c_int, vp]
    L.qmm_moe_gemm_id.restype = c_int
    L.qmm_moe_gemm_id_noalloc.argtypes = [vp, c_int, vp, i64, i64, i64, stp, vp, c_int, vp, vp]
    L.qmm_moe_gemm_id_noalloc.restype = c_int
    L.qmm_selftest_bounded_wait.argtypes = [ctypes.c_uint32, vp, vp, vp]
    L.qmm_selftest_bounded_wait.restype = c_int
    L.qmm_matmul_parts.argtypes = [vp, c_int, i64, i64, qwp, c_int, vp, c_int, vp]
    L.qmm_matmul_parts.restype = c_int
    L.qmm_quantize_dynamic_int8.argtypes = [vp, c_int, i64, vp, vp, vp]
    L.qmm_quantize_dynamic_int8.restype = c_int
    L.qmm_dequantize_dynamic_int8.argtypes = [vp, i64, vp, vp, c_int, vp]
    L.qmm_dequantize_dynamic_int8.restype = c_int
    L.qmm_matmul_dynamic_int8.argtypes = [vp, c_int, i64, i64, vp, i64, vp, vp, c_int, vp]
    L.qmm_matmul_dynamic_int8.restype = c_int
    _lib = L
    return L


def status_string(code: int) -> str:
    return load().qmm_status_string(int(code)).decode()


class QmmError(RuntimeError):
    def __init__(self, call: str, code: int):
        self.code = int(code)
        super().__init__(f"{call} failed: {status_string(code)} (status {code})")


def check(call: str, code: int) -> None:
    if code != QMM_OK:
        raise QmmError(call, code)
