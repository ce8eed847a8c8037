"""Shared helpers of the parity tests: moving tensors to oracle (numpy storage)
form and the tolerance gates."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from weight_only_quantized_qmm_b200 import workloads as wl

ORC = {torch.float32: oracle.F32, torch.float16: oracle.F16, torch.bfloat16: oracle.BF16}

# spec gates for matmul-type outputs against the fp64 oracle
REL_FRO = 5e-3
MAX_ABS_RMS = 1e-2


def np_storage(t: torch.Tensor) -> np.ndarray:
    return wl.storage_numpy(t.detach().cpu())


def packed_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def qweight_np(qw):
    return packed_np(qw.packed), np_storage(qw.scales), np_storage(qw.biases)


def gate(y: np.ndarray, yref: np.ndarray, what: str = ""):
    """rel-Frobenius <= 5e-3 and max|y - yref| <= 1e-2 * rms(yref)."""
    y = np.asarray(y, dtype=np.float64)
    yref = np.asarray(yref, dtype=np.float64)
    assert y.shape == yref.shape, (y.shape, yref.shape)
    err = y - yref
    nref = np.linalg.norm(yref)
    rms = np.sqrt(np.mean(yref ** 2)) if yref.size else 0.0
    rel = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= REL_FRO, f"{what}: rel-Frobenius {rel:.3e} > {REL_FRO}"
    assert mx <= MAX_ABS_RMS * rms + 1e-30, f"{what}: max-abs {mx:.3e} > {MAX_ABS_RMS}*rms({rms:.3e})"
    return rel, mx / rms if rms else 0.0


def rne_equal(y16: torch.Tensor, y32: torch.Tensor):
    """16-bit output must equal RNE of the same kernel's fp32 output."""
    ref = y32.to(y16.dtype)
    a = y16.view(torch.int16).cpu()
    b = ref.view(torch.int16).cpu()
    assert torch.equal(a, b), f"{int((a != b).sum())} elements differ from RNE(fp32 result)"
