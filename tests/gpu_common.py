"""Helpers shared by the GPU parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16 / fp32 / fp64 tensor (on any device)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return fp64.bf16_bits_to_f64(synth.bf16_bits(t))
    return t.to(torch.float64).numpy()


def same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    """Bitwise equality (NaN-safe, distinguishes -0 from +0)."""
    if a.shape != b.shape or a.dtype != b.dtype:
        return False
    a = a.detach().contiguous()
    b = b.detach().contiguous()
    ia = a.view(torch.int16) if a.element_size() == 2 else a.view(torch.int32)
    ib = b.view(torch.int16) if b.element_size() == 2 else b.view(torch.int32)
    return bool(torch.equal(ia, ib))


def dev(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda:0").contiguous()
