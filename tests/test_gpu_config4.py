"""Dense decoder at the Mistral-7B shape (32 layers, d 4096, 32/8 GQA heads,
FFN 14336 SwiGLU, RoPE theta 1e4, vocab 32000), random-init bf16 weights
(std 0.02, norms 1, seed 0): a 1400-token prompt of uniform random token ids
(seed 1) decoded greedily for 128 tokens, alone and co-batched with 1, 7 and
63 other prompts of lengths uniform in [16, 2048] under a seeded scheduler
that varies chunk sizes -- the request's logits (fp32) and tokens must be the
same bits every time ("Defeating Nondeterminism in LLM Inference", section
"Batch invariance and determinism": a request's output must not depend on
the server's load). A short teacher-forced prefix is also checked against
the fp64 oracle in the fp32-activation mode."""
import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64
from tests.gpu_common import f64, same_bits

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CFG = dict(n_layers=32, d_model=4096, n_q_heads=32, n_kv_heads=8, d_ff=14336, vocab=32000,
           max_pos=4096, rms_eps=1e-6, rope_theta=1e4)
PROMPT, NEW = 1400, 128


@pytest.fixture(scope="module")
def weights():
    w = synth.model_weights(CFG, seed=0)
    return w, {k: v.cuda().contiguous() for k, v in w.items()}


def _engine(cfg, wd, seed, max_tokens, pages=10240):
    from invariant_deterministic_03_b200 import runner
    return runner.Engine(cfg, wd, num_pages=pages, max_pages_per_seq=cfg["max_pos"] // 16,
                         max_tokens=max_tokens, max_logits=64, seed=seed)


def _serve(cfg, wd, others, sched_seed, engine_seed):
    """Run request 0 (the prompt) plus `others` through one engine; each step
    takes every live request, prefill chunks drawn from a seeded choice of
    sizes. Returns request 0's logits rows [1 + NEW, V] and its new tokens."""
    rng = np.random.default_rng(sched_seed)
    prompt = synth.randint(PROMPT, 0, cfg["vocab"] - 1, seed=1).tolist()
    reqs = {0: {"toks": list(prompt), "plen": PROMPT, "new": 0}}
    for i, toks in enumerate(others):
        reqs[i + 1] = {"toks": list(toks), "plen": len(toks), "new": 0}
    eng = _engine(cfg, wd, engine_seed, max_tokens=8192)
    done = {s: 0 for s in reqs}
    logits0, toks0 = [], []
    sizes = [16, 64, 128, 512, 1024, 2048]
    while reqs[0]["new"] < NEW:
        chunks, budget = [], 8192
        order = list(reqs)
        rng.shuffle(order)                      # batch position varies step to step
        for s in order:
            r = reqs[s]
            if r["new"] >= NEW and s != 0:
                continue
            if done[s] < r["plen"]:
                n = min(int(rng.choice(sizes)), r["plen"] - done[s], budget)
            else:
                n = 1 if budget > 0 else 0
            if n <= 0:
                continue
            chunks.append((s, done[s], done[s] + n))
            budget -= n
        lg, nxt = eng.step(chunks, lambda s: reqs[s]["toks"])
        nxt = nxt.tolist()
        for i, (s, a, b) in enumerate(chunks):
            done[s] = b
            r = reqs[s]
            if b == len(r["toks"]) and b >= r["plen"]:      # this chunk ended the known tokens
                if s == 0:
                    logits0.append(lg[i].clone())
                    toks0.append(nxt[i])
                if r["new"] < NEW:
                    r["toks"].append(nxt[i])
                    r["new"] += 1
        reqs = {s: r for s, r in reqs.items() if s == 0 or r["new"] < NEW}
    return torch.stack(logits0), toks0


def test_config4_bitwise_across_cobatching(weights):
    _, wd = weights
    ref_logits, ref_toks = _serve(CFG, wd, [], sched_seed=100, engine_seed=0)
    assert len(ref_toks) == NEW and ref_logits.shape == (NEW, CFG["vocab"])
    assert torch.isfinite(ref_logits).all()
    for k, seed in [(1, 2), (7, 3), (63, 4)]:
        lens = synth.randint(k, 16, 2048, seed=seed).tolist()
        others = [synth.randint(L, 0, CFG["vocab"] - 1, seed=seed * 1000 + i).tolist()
                  for i, L in enumerate(lens)]
        lg, tk = _serve(CFG, wd, others, sched_seed=seed, engine_seed=seed)
        assert tk == ref_toks, f"{k} co-batched requests: tokens differ"
        assert same_bits(lg, ref_logits), f"{k} co-batched requests: logits differ"
    # run to run
    lg, tk = _serve(CFG, wd, [], sched_seed=100, engine_seed=0)
    assert tk == ref_toks and same_bits(lg, ref_logits)


def test_config4_fp32_mode_prefix_vs_fp64(weights):
    """fp32-activation mode, teacher forced on the first 24 prompt tokens:
    max |logit - fp64| <= 1e-2 at the full 32-layer depth."""
    w, wd = weights
    cfg = dict(CFG, precision="f32")
    n = 24
    toks = synth.randint(PROMPT, 0, CFG["vocab"] - 1, seed=1).tolist()[:n]
    eng = _engine(cfg, wd, seed=9, max_tokens=256, pages=64)
    lg = torch.cat([eng.step([(0, p, p + 1)], lambda s: toks)[0] for p in range(n)])
    ref = fp64.forward(fp64.ModelWeights(CFG, {k: synth.bf16_bits(v) for k, v in w.items()}), toks)
    err = np.abs(f64(lg) - ref)
    assert err.max() <= 1e-2, f"max abs logit error {err.max():.3e}"
