"""The FP16 variant of the cross-vendor paper's precision study (arXiv
2610.05458, abstract): the bf16 forward with fp16 in place of bf16 for the
weights, activations, KV cache and attention's P. Its logits against the
fp64 oracle (teacher forced, the model's fp16 weights), bounded by 1.5x the
error of the fp64 forward with fp16 storage at the same points; and the same
batch invariance as the bf16 path: decode == chunked prefill == co-batched,
bitwise."""
import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64
from tests.gpu_common import all_position_logits, emulated_logit_bounds, f64, same_bits

pytestmark = pytest.mark.gpu

SMALL = dict(n_layers=2, d_model=256, n_q_heads=2, n_kv_heads=1, d_ff=384, vocab=512,
             max_pos=2048, rms_eps=1e-6, rope_theta=1e4, precision="f16")
MID = dict(n_layers=2, d_model=4096, n_q_heads=32, n_kv_heads=8, d_ff=14336, vocab=32000,
           max_pos=4096, rms_eps=1e-6, rope_theta=1e4, precision="f16")


def _engine(cfg, w16, seed, max_tokens=1024, max_logits=1024, pages=1024):
    from invariant_deterministic_03_b200 import runner
    wd = {k: v.cuda().contiguous() for k, v in w16.items()}
    return runner.Engine(cfg, wd, num_pages=pages, max_pages_per_seq=cfg["max_pos"] // 16,
                         max_tokens=max_tokens, max_logits=max_logits, seed=seed)


@pytest.mark.parametrize("cfg,n", [(SMALL, 600), (MID, 40)], ids=["small-600", "mistral-shape-2-layers"])
def test_f16_forward_vs_fp64(cuda_device, cfg, n):
    w16 = synth.to_f16(synth.model_weights(cfg, seed=3))
    toks = synth.randint(n, 0, cfg["vocab"] - 1, seed=4).tolist()
    lg = all_position_logits(_engine(cfg, w16, seed=0), toks, 256)
    ow = fp64.ModelWeights(cfg, {k: synth.bf16_bits(v) for k, v in w16.items()}, fmt="f16")
    ref = fp64.forward(ow, toks)
    max_abs, grel, emu = emulated_logit_bounds(ow, toks, "f16", ref)
    err = np.abs(f64(lg) - ref)
    assert err.max() <= max_abs, f"max abs logit error {err.max():.3e} (emulated {emu['max_abs']:.3e})"
    assert np.linalg.norm(f64(lg) - ref) <= grel * np.linalg.norm(ref)


def test_f16_decode_prefill_cobatch_bitwise(cuda_device):
    cfg = SMALL
    w16 = synth.to_f16(synth.model_weights(cfg, seed=5))
    n = 700
    toks = synth.randint(n, 0, cfg["vocab"] - 1, seed=6).tolist()
    whole = all_position_logits(_engine(cfg, w16, seed=1), toks, 700)
    chunked = all_position_logits(_engine(cfg, w16, seed=2), toks, 64)
    assert same_bits(whole, chunked)
    # decode steps past the 512-key split, co-batched with another request
    eng = _engine(cfg, w16, seed=3)
    other = synth.randint(300, 0, cfg["vocab"] - 1, seed=7).tolist()
    tok_of = lambda s: toks if s == 0 else other   # noqa: E731
    all_position_logits(eng, toks[:600], 300)
    eng.step([(1, 0, 200)], tok_of)
    for p in range(600, 606):
        lg, _ = eng.step([(1, 200 + p - 600, 201 + p - 600), (0, p, p + 1)], tok_of)
        assert same_bits(lg[1], whole[p]), f"position {p}"
