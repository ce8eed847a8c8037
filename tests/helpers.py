"""Shared helpers of the parity tests: moving tensors to oracle (numpy storage)
form, the tolerance gates, guarded output buffers and the worst-case record."""
from __future__ import annotations

import json
import os
import threading

import numpy as np
import torch

import oracle
from weight_only_quantized_qmm_b200 import workloads as wl

ORC = {torch.float32: oracle.F32, torch.float16: oracle.F16, torch.bfloat16: oracle.BF16}

# spec gates for matmul-type outputs against the fp64 oracle
REL_FRO = 5e-3
MAX_ABS_RMS = 1e-2

# worst observed (rel-Frobenius, max-abs / rms) per gate label; written as JSON
# at the end of the session when QMM_PARITY_REPORT names a file
_WORST: dict = {}
_WLOCK = threading.Lock()


def record(what: str, rel: float, ratio: float, n: int) -> None:
    with _WLOCK:
        old = _WORST.get(what)
        if old is None or ratio > old["max_abs_over_rms"]:
            _WORST[what] = {"rel_fro": float(rel), "max_abs_over_rms": float(ratio), "outputs": int(n)}


def write_report() -> None:
    path = os.environ.get("QMM_PARITY_REPORT")
    if path and _WORST:
        os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
        with open(path, "w") as f:
            json.dump({"gate": {"rel_fro": REL_FRO, "max_abs_over_rms": MAX_ABS_RMS},
                       "worst": _WORST}, f, indent=1, sort_keys=True)


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
    assert np.all(np.isfinite(y)), f"{what}: {int((~np.isfinite(y)).sum())} non-finite outputs"
    err = y - yref
    nref = np.linalg.norm(yref)
    rms = np.sqrt(np.mean(yref ** 2)) if yref.size else 0.0
    rel = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    mx = np.abs(err).max() if err.size else 0.0
    ratio = mx / rms if rms else 0.0
    record(what, rel, ratio, y.size)
    assert rel <= REL_FRO, f"{what}: rel-Frobenius {rel:.3e} > {REL_FRO}"
    assert mx <= MAX_ABS_RMS * rms + 1e-30, f"{what}: max-abs {mx:.3e} > {MAX_ABS_RMS}*rms({rms:.3e})"
    return rel, ratio


def rne_equal(y16: torch.Tensor, y32: torch.Tensor):
    """16-bit output must equal RNE of the same kernel's fp32 output."""
    ref = y32.to(y16.dtype)
    a = y16.view(torch.int16).cpu()
    b = ref.view(torch.int16).cpu()
    assert torch.equal(a, b), f"{int((a != b).sum())} elements differ from RNE(fp32 result)"


# ------------------------------------------------------------------ guarded outputs
GUARD = 4096  # elements of guard band after every guarded output
# NaN bit patterns no kernel writes (quiet NaN with a payload)
_POISON = {torch.float32: (torch.int32, 0x7FC0DEAD), torch.float16: (torch.int16, 0x7E5A),
           torch.bfloat16: (torch.int16, 0x7FDA)}


class Guarded:
    """An output tensor poisoned with a NaN pattern and followed by a guard band
    of the same pattern: after the call every output element must have been
    written (no poison left) and the guard band must be untouched."""

    def __init__(self, shape, dtype, device="cuda"):
        n = int(np.prod(shape))
        idt, pat = _POISON[dtype]
        raw = torch.full((n + GUARD,), pat, dtype=idt, device=device)  # positive: fits idt
        self.raw = raw
        self.pat = raw[-1].item()
        self.n = n
        self.buf = raw.view(dtype)
        self.out = self.buf[:n].view(*shape)

    def check(self, what=""):
        raw = self.raw.cpu()
        left = int((raw[:self.n] == self.pat).sum())
        assert left == 0, f"{what}: {left} output elements never written"
        hit = int((raw[self.n:] != self.pat).sum())
        assert hit == 0, f"{what}: {hit} guard-band elements past the output were overwritten"
        return self.out
