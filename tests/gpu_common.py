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


# Tolerance of a mixed-precision forward's logits against the fp64 oracle:
# the fp64 forward with the mode's storage roundings (fp64.forward_rounded)
# shows how far those roundings alone move the logits; the GPU path rounds at
# the same points but accumulates in fp32 in its own order, so its error is
# of the same size, not the same values. Bound = EMULATED_MARGIN x the
# emulated error (max abs and global relative alike).
EMULATED_MARGIN = 1.5


def emulated_logit_bounds(weights, tokens, mode, ref=None):
    """(max_abs, global_rel) bounds for `mode` from the rounding emulation,
    and the emulated errors themselves."""
    if ref is None:
        ref = fp64.forward(weights, tokens)
    emu = fp64.forward_rounded(weights, tokens, mode)
    e_max = float(np.max(np.abs(emu - ref)))
    e_rel = float(np.linalg.norm(emu - ref) / np.linalg.norm(ref))
    return EMULATED_MARGIN * e_max, EMULATED_MARGIN * e_rel, {"max_abs": e_max, "global_rel": e_rel}


def all_position_logits(eng, toks, chunk, seq=0, start=0):
    """Feed toks[start:] to sequence `seq` of an engine in chunks, with a
    logits row for EVERY position (the engine's steps return only each
    chunk's last row). Returns [len(toks) - start, V] fp32 on the device."""
    from invariant_deterministic_03_b200 import runner
    out = []
    for s in range(start, len(toks), chunk):
        e = min(len(toks), s + chunk)
        b = runner.make_batch(eng.kv, [(seq, s, e)], lambda _s: toks)
        b["max_kv_len"] = eng.cfg["max_pos"]
        b["logits_rows"] = torch.arange(e - s, dtype=torch.int32, device="cuda:0")
        lg = torch.empty(e - s, eng.cfg["vocab"], dtype=torch.float32, device="cuda:0")
        eng.model.forward(b, eng.kv.k, eng.kv.v, lg, None, eng.ws)
        runner.commit(eng.kv, [(seq, s, e)])
        out.append(lg)
    return torch.cat(out)
