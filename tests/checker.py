"""Tolerance rule used by every parity test (independent of both the oracle's
arithmetic and the CUDA path).

"GPU program deployment: verifying correctness" (sections on evaluation blind
spots and on verification) warns that a tolerance far above the size of the
output lets wrong programs pass (its softmax example: an all-zero output passes
a 0.01 tolerance when outputs are ~2.5e-6) and asks for several independent
checks: shape, NaN/Inf, absolute and relative error scaled to the data, and
error versus problem size. The rule here:

  per element  |y - y64| <= rel * |y64| + rel * kappa * R
  globally     ||y - y64||_2 <= grel * ||y64||_2

rel = 2^-7 (one bf16 output rounding is 2^-9 relative, so this leaves a
factor of 4), R = sqrt(sum_j t_j^2) over the terms t_j the element reduces
(the natural size of a cancelling sum), kappa per operation: 1/16 for the
GEMM (fp32 accumulation only), 1 for attention (bf16 rounding of the softmax
weights), 0 for RMSNorm (no cancellation).
"""
from __future__ import annotations

import numpy as np

REL = 2.0 ** -7
GLOBAL_REL = 2.0 ** -8


class ParityError(AssertionError):
    pass


def check(y, y64, R=None, kappa: float = 0.0, rel: float = REL,
          global_rel: float = GLOBAL_REL, what: str = "") -> dict:
    y = np.asarray(y, dtype=np.float64)
    y64 = np.asarray(y64, dtype=np.float64)
    if y.shape != y64.shape:
        raise ParityError(f"{what}: shape {y.shape} != {y64.shape}")
    if not np.all(np.isfinite(y)):
        bad = np.argwhere(~np.isfinite(y))[:5].tolist()
        raise ParityError(f"{what}: non-finite outputs at {bad}")
    err = np.abs(y - y64)
    bound = rel * np.abs(y64)
    if R is not None and kappa:
        bound = bound + rel * kappa * np.asarray(R, dtype=np.float64)
    viol = err > bound
    report = {
        "what": what,
        "n": int(y.size),
        "max_abs_err": float(err.max()) if err.size else 0.0,
        "max_rel_err": float((err / np.maximum(np.abs(y64), 1e-300)).max()) if err.size else 0.0,
        "violations": int(viol.sum()),
        "needed_kappa_term": int(np.sum(err > rel * np.abs(y64))),
    }
    if viol.any():
        idx = np.argwhere(viol)[:5]
        detail = [(tuple(i), float(y[tuple(i)]), float(y64[tuple(i)]), float(bound[tuple(i)])) for i in idx]
        raise ParityError(f"{what}: {report['violations']} elements out of tolerance, e.g. {detail}")
    n64 = float(np.linalg.norm(y64))
    gerr = float(np.linalg.norm(y - y64))
    report["global_rel_err"] = gerr / n64 if n64 else gerr
    if n64 and gerr > global_rel * n64:
        raise ParityError(f"{what}: global relative error {gerr / n64:.3e} > {global_rel:.3e}")
    if not n64 and gerr:
        raise ParityError(f"{what}: expected all zeros, got norm {gerr:.3e}")
    return report
