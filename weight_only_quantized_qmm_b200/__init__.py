"""Weight-only quantized matmul for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``lib/libqmm.so`` (declared in
``include/qmm.h``); this package is its Python binding (``api``), the in-tree
build (``build``) and the seeded synthetic workloads (``workloads``).
"""
from .api import (ExpertStack, QWeight, qmm_dequantize, qmm_device_check, qmm_groups_per_row,
                  qmm_matmul, qmm_moe_gemv_id, qmm_moe_gemv_id_batched,
                  qmm_moe_gemv_id_gate_up_silu, qmm_moe_gemv_id_gate_up_silu_batched,
                  qmm_packed_words_per_row, qmm_quantize, qmm_status_string)

__all__ = [
    "ExpertStack", "QWeight", "qmm_dequantize", "qmm_device_check", "qmm_groups_per_row",
    "qmm_matmul", "qmm_moe_gemv_id", "qmm_moe_gemv_id_batched", "qmm_moe_gemv_id_gate_up_silu",
    "qmm_moe_gemv_id_gate_up_silu_batched", "qmm_packed_words_per_row", "qmm_quantize",
    "qmm_status_string",
]
