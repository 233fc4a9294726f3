"""Seeded synthetic inputs for Sparse-BitLinear.

This module only draws random numbers; it holds none of the operator's
arithmetic, so both the CUDA path and the CPU oracle may take their inputs
from it.  Distributions follow the workloads of the Sparse-BitNet experiments
as restated for this library: master weights ~ N(0, 0.02) and activations /
upstream gradients ~ N(0, 1), drawn in fp32 and rounded to bf16.
"""
from __future__ import annotations

import torch

WEIGHT_STD = 0.02


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from a generator seeded with ``seed``, rounded to bf16."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    v = torch.randn(tuple(shape), generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        v = v * std
    return v.to(torch.bfloat16)


def master_weights(n_out: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [n_out, k] master weights ~ N(0, 0.02)."""
    return normal_bf16((n_out, k), WEIGHT_STD, seed, device)


def activations(t: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [t, k] activations ~ N(0, 1)."""
    return normal_bf16((t, k), 1.0, seed, device)


def upstream_grad(t: int, n_out: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [t, n_out] upstream gradient ~ N(0, 1)."""
    return normal_bf16((t, n_out), 1.0, seed, device)


def bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor's bit patterns (copied to host)."""
    import numpy as np

    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
