"""Seeded synthetic inputs for the group-wise low-bit linear workloads.

This module only draws random numbers with fixed seeds; it holds none of the
method's arithmetic (no quantization, packing or dequantization).  Both the
tests (which feed the CPU oracle and the CUDA library the same inputs) and the
benchmark use it.

Recipes (all on a CPU ``torch.Generator`` so values are identical everywhere):
  * weights:      fp32 N(0, 0.02) [N, K], seed 0
  * activations:  N(0, 1) [M, K], seed 1, optionally a fraction of input
                  channels (chosen by a seeded randperm, seed 2) multiplied by
                  an outlier factor (x20) for every token
  * GPTQ quartet: qweight / qzeros as uniformly random 32-bit words (so every
                  4-bit field is uniform in [0, 15]), fp16 scales uniform in
                  [0.001, 0.02], seed 0; g_idx = i // gs, or a seeded shuffle
                  (seed 3) of that vector (every group keeps gs members)
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weights(N: int, K: int, seed: int = 0, std: float = 0.02) -> torch.Tensor:
    """fp32 [N, K] ~ N(0, std^2)."""
    return torch.randn((N, K), generator=_gen(seed), dtype=torch.float32) * std


def activations(M: int, K: int, seed: int = 1, dtype=torch.bfloat16,
                outlier_frac: float = 0.0, outlier_scale: float = 20.0,
                outlier_seed: int = 2) -> torch.Tensor:
    """[M, K] ~ N(0, 1) in `dtype`; round(outlier_frac*K) channels scaled by outlier_scale."""
    x = torch.randn((M, K), generator=_gen(seed), dtype=torch.float32)
    n_out = int(round(outlier_frac * K))
    if n_out:
        ch = torch.randperm(K, generator=_gen(outlier_seed))[:n_out]
        x[:, ch] *= outlier_scale
    return x.to(dtype)


def random_words(shape, seed: int) -> torch.Tensor:
    """int32 tensor of uniformly random 32-bit patterns."""
    g = _gen(seed)
    lo = torch.randint(0, 1 << 16, shape, generator=g, dtype=torch.int64)
    hi = torch.randint(0, 1 << 16, shape, generator=g, dtype=torch.int64)
    u = (hi << 16) | lo
    return (u - ((u >> 31) << 32)).to(torch.int32)


def gptq_quartet(K: int, N: int, gs: int, seed: int = 0, permuted: bool = False,
                 perm_seed: int = 3):
    """(qweight int32 [K/8, N], scales fp16 [K/gs, N], qzeros int32 [K/gs, N/8], g_idx int32 [K])."""
    qweight = random_words((K // 8, N), seed)
    qzeros = random_words((K // gs, N // 8), seed + 1000)
    u = torch.rand((K // gs, N), generator=_gen(seed + 2000), dtype=torch.float32)
    scales = (0.001 + u * (0.02 - 0.001)).to(torch.float16)
    g_idx = torch.arange(K, dtype=torch.int64) // gs
    if permuted:
        g_idx = g_idx[torch.randperm(K, generator=_gen(perm_seed))]
    return qweight, scales, qzeros, g_idx.to(torch.int32)


def bits16(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16 / fp16 tensor as np.uint16 (a view, no rounding)."""
    assert t.dtype in (torch.bfloat16, torch.float16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits16(a: np.ndarray, dtype) -> torch.Tensor:
    """Inverse of bits16."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dtype)
