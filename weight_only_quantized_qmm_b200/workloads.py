"""Seeded synthetic inputs for the quantized-matmul workloads.

This module holds no arithmetic of the method itself: it only draws random
inputs (dense weights, activations, expert ids) with a seeded CPU torch
generator and names the workload shapes.  Both the CUDA path (through the
package API) and the CPU oracle consume exactly these bytes.

Recipe (the same for every workload):
  * W  = 0.02 * randn(N, K) in fp32 (then quantized by the library);
  * x  = randn(M, K) in fp32, cast to bf16 with round-to-nearest-even;
  * MoE ids: for each token, randperm(E)[:top_k] (distinct, uniform) as int32.
Seeds: seed 0 for the tiny case; otherwise 1000*workload_index + variant.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def gen_weight(n: int, k: int, seed: int, std: float = 0.02) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randn(n, k, generator=g, dtype=torch.float32) * std


def gen_x(m: int, k: int, seed: int, dtype: str = "bf16") -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randn(m, k, generator=g, dtype=torch.float32).to(_DT[dtype])


def gen_moe_ids(tokens: int, num_experts: int, top_k: int, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    ids = torch.stack([torch.randperm(num_experts, generator=g)[:top_k] for _ in range(tokens)])
    return ids.to(torch.int32).contiguous()


def storage_numpy(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a CPU tensor in storage form (uint16 bits for 16-bit floats)."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def iota(rows: int, cols: int, dtype=torch.float32) -> torch.Tensor:
    """Nx.iota({rows, cols}): 0, 1, 2, ... in row-major order."""
    return torch.arange(rows * cols, dtype=torch.float64).reshape(rows, cols).to(dtype)


@dataclass
class DenseCase:
    name: str
    M: int
    N: int
    K: int
    bits: int = 4
    group_size: int = 64
    seed: int = 0


@dataclass
class MoECase:
    name: str
    tokens: int
    num_experts: int = 128
    top_k: int = 8
    d_model: int = 2048
    d_ff: int = 768
    bits: int = 4
    group_size: int = 64
    seed: int = 0


@dataclass
class Workloads:
    tiny: DenseCase = field(default_factory=lambda: DenseCase("tiny", 4, 256, 512, 4, 64, 0))
    decode: list = field(default_factory=lambda: [
        DenseCase("decode_4096x4096", 1, 4096, 4096, 4, 64, 1000),
        DenseCase("decode_14336x4096", 1, 14336, 4096, 4, 64, 1001),
        DenseCase("decode_4096x14336", 1, 4096, 14336, 4, 64, 1002),
    ])
    sweep: list = field(default_factory=lambda: [
        DenseCase(f"sweep_b{b}_g{g}_m{m}", m, 8192, 8192, b, g, 2000 + 100 * b + g + m)
        for b in (2, 3, 6, 8) for g in (32, 64, 128) for m in (1, 4, 16)
    ])
    prefill: list = field(default_factory=lambda: [
        DenseCase(f"prefill_m{m}_{n}x{k}", m, n, k, 4, 64, 3000 + i)
        for i, (m, (n, k)) in enumerate((m, nk) for nk in ((4096, 4096), (14336, 4096))
                                         for m in (512, 2048, 4096))
    ])
    moe: list = field(default_factory=lambda: [
        MoECase(f"moe_t{t}", t, seed=4000 + t) for t in (1, 16, 64)
    ])


WORKLOADS = Workloads()
