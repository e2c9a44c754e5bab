"""Prefix caching with invariant reuse: a request that starts from another
request's cached prefix pages gives the same logits and greedy tokens,
bitwise, as computing its whole prompt itself ("Defeating Nondeterminism in
LLM Inference", section "Batch-invariant attention": keys are reduced at the
same absolute tile and split boundaries whether they were cached earlier or
belong to the chunk in flight)."""
import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64
from tests.gpu_common import emulated_logit_bounds, f64, same_bits

pytestmark = pytest.mark.gpu

SMALL = dict(n_layers=2, d_model=256, n_q_heads=2, n_kv_heads=1, d_ff=384, vocab=512,
             max_pos=2048, rms_eps=1e-6, rope_theta=1e4)
MID = dict(n_layers=2, d_model=4096, n_q_heads=32, n_kv_heads=8, d_ff=14336, vocab=32000,
           max_pos=4096, rms_eps=1e-6, rope_theta=1e4)


def _engine(cfg, wd, seed):
    from invariant_deterministic_03_b200 import runner
    return runner.Engine(cfg, wd, num_pages=512, max_pages_per_seq=cfg["max_pos"] // 16,
                         max_tokens=1024, max_logits=8, seed=seed)


def _prefill_then_decode(eng, seq, toks, start, chunks, n_new):
    """Feeds toks[start:] in the given chunk sizes, then decodes n_new tokens
    greedily; returns the logits rows (one per step) and the new tokens."""
    toks = list(toks)
    rows, pos = [], start
    for c in chunks:
        e = min(len(toks), pos + c)
        if e <= pos:
            break
        lg, nxt = eng.step([(seq, pos, e)], lambda _s: toks)
        pos = e
    rows.append(lg[0].clone())
    toks.append(int(nxt[0]))
    for _ in range(n_new - 1):
        lg, nxt = eng.step([(seq, len(toks) - 1, len(toks))], lambda _s: toks)
        rows.append(lg[0].clone())
        toks.append(int(nxt[0]))
    return torch.stack(rows), toks[-n_new:]


@pytest.mark.parametrize("cfg,prefix,suffix", [(SMALL, 200, 37), (MID, 523, 60)], ids=["small", "mistral-shape"])
def test_prefix_reuse_is_bitwise(cuda_device, cfg, prefix, suffix):
    w = synth.model_weights(cfg, seed=21)
    wd = {k: v.cuda().contiguous() for k, v in w.items()}
    shared = synth.randint(prefix, 0, cfg["vocab"] - 1, seed=22).tolist()
    a_toks = shared + synth.randint(25, 0, cfg["vocab"] - 1, seed=23).tolist()
    b_toks = shared + synth.randint(suffix, 0, cfg["vocab"] - 1, seed=24).tolist()

    # B alone, whole prompt computed by itself
    ref_rows, ref_new = _prefill_then_decode(_engine(cfg, wd, seed=1), 0, b_toks, 0, [64] * 64, 6)

    # A first, then B forks A's cached prefix pages and computes only the rest
    eng = _engine(cfg, wd, seed=2)
    _prefill_then_decode(eng, 0, a_toks, 0, [128] * 64, 2)
    held = eng.kv.fork(0, 1, prefix)
    assert held == (prefix // 16) * 16 and held > 0
    assert eng.kv.pages[1] == eng.kv.pages[0][: held // 16]      # the same physical pages
    rows, new = _prefill_then_decode(eng, 1, b_toks, held, [17, 128, 1024], 6)
    assert new == ref_new
    assert same_bits(rows, ref_rows)
    # and against the fp64 oracle, teacher forced on the forked request's
    # tokens: row i is the logits at position len(b_toks) - 1 + i
    seq = b_toks + new[:-1]
    ow = fp64.ModelWeights(cfg, {k: synth.bf16_bits(v) for k, v in w.items()})
    ref = fp64.forward(ow, seq)
    max_abs, _, emu = emulated_logit_bounds(ow, seq, "bf16", ref)
    err = np.max(np.abs(f64(rows) - ref[len(b_toks) - 1:]))
    assert err <= max_abs, f"max abs logit error {err:.3e} (emulated {emu['max_abs']:.3e})"

    # releasing the source keeps the shared pages alive for the fork
    eng.kv.release(0)
    assert all(eng.kv.refs[p] == 1 for p in eng.kv.pages[1])
    rows2, _ = _prefill_then_decode(eng, 1, b_toks + new, len(b_toks) + len(new) - 1, [1], 1)
    assert torch.isfinite(rows2).all()
