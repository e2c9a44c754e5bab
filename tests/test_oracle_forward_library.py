"""The oracle against independent library implementations, on the CPU (no
GPU, no network): its decoder forward against the Mistral model of the
`transformers` library run in float64 with the same weights, its attention
against torch's float64 scaled_dot_product_attention, and its RMSNorm
against torch's rms_norm.

The forward the oracle writes out (pre-norm RMSNorm, rotate-half RoPE with
theta 1e4 at absolute positions, grouped-query causal attention with q head
h reading kv head h // (Hq / Hkv), SwiGLU MLP, final RMSNorm, untied LM head)
is the architecture of the model the pages run (Mistral-7B). A mistake in
any step of the oracle's composition -- a transposed projection, the wrong
RoPE pairing or sign, the wrong head grouping, a misplaced norm, gate and up
swapped -- moves logits by O(1); the library computes its RMSNorm variance and
its RoPE angles in float32 even in a float64 model, so agreement is to
~1e-6, and the bound below is 1e-4.
"""
import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64

transformers = pytest.importorskip("transformers")

CFG = dict(n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=2, d_ff=384, vocab=512,
           max_pos=256, rms_eps=1e-6, rope_theta=1e4)


def _weights():
    w = synth.model_weights(CFG, seed=7, std=0.05)
    # norms away from one, so the gamma multiplications are pinned too
    L, D = CFG["n_layers"], CFG["d_model"]
    w["attn_norm"] = synth.uniform_bf16((L, D), 0.5, 1.5, 71)
    w["mlp_norm"] = synth.uniform_bf16((L, D), 0.5, 1.5, 72)
    w["final_norm"] = synth.uniform_bf16((D,), 0.5, 1.5, 73)
    return w


def _library_model(w):
    c = CFG
    conf = transformers.MistralConfig(
        vocab_size=c["vocab"], hidden_size=c["d_model"], intermediate_size=c["d_ff"],
        num_hidden_layers=c["n_layers"], num_attention_heads=c["n_q_heads"],
        num_key_value_heads=c["n_kv_heads"], head_dim=128, max_position_embeddings=c["max_pos"],
        rms_norm_eps=c["rms_eps"], rope_theta=c["rope_theta"], sliding_window=None,
        tie_word_embeddings=False, attn_implementation="eager")
    m = transformers.MistralForCausalLM(conf).double().eval()
    hq, hkv, F = c["n_q_heads"] * 128, c["n_kv_heads"] * 128, c["d_ff"]
    f64 = lambda t: t.to(torch.float64)  # noqa: E731  (bf16 -> float64 is exact)
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(f64(w["embed"]))
        m.lm_head.weight.copy_(f64(w["lm_head"]))
        m.model.norm.weight.copy_(f64(w["final_norm"]))
        for l, layer in enumerate(m.model.layers):
            qkv = f64(w["w_qkv"][l])
            layer.self_attn.q_proj.weight.copy_(qkv[:hq])
            layer.self_attn.k_proj.weight.copy_(qkv[hq:hq + hkv])
            layer.self_attn.v_proj.weight.copy_(qkv[hq + hkv:])
            layer.self_attn.o_proj.weight.copy_(f64(w["w_o"][l]))
            gu = f64(w["w_gate_up"][l])
            layer.mlp.gate_proj.weight.copy_(gu[:F])
            layer.mlp.up_proj.weight.copy_(gu[F:])
            layer.mlp.down_proj.weight.copy_(f64(w["w_down"][l]))
            layer.input_layernorm.weight.copy_(f64(w["attn_norm"][l]))
            layer.post_attention_layernorm.weight.copy_(f64(w["mlp_norm"][l]))
    return m


def test_oracle_forward_matches_library_mistral():
    w = _weights()
    tokens = synth.randint(48, 0, CFG["vocab"] - 1, seed=8).tolist()
    ours = fp64.forward(fp64.ModelWeights(CFG, {k: synth.bf16_bits(v) for k, v in w.items()}), tokens)
    with torch.no_grad():
        lib = _library_model(w)(torch.tensor([tokens])).logits[0].numpy()
    assert ours.shape == lib.shape
    scale = np.abs(lib).max()
    assert scale > 0.1                       # logits of a real size, not a degenerate model
    err = np.abs(ours - lib).max()
    assert err <= 1e-4, f"max |oracle - library| = {err:.3e} (logit scale {scale:.3f})"


def test_library_comparison_catches_a_planted_mistake():
    """Swap gate and up in the oracle's weights (a plausible mistake): the
    comparison must fail by far more than its bound."""
    w = _weights()
    tokens = synth.randint(16, 0, CFG["vocab"] - 1, seed=9).tolist()
    F = CFG["d_ff"]
    bad = dict(w)
    bad["w_gate_up"] = torch.cat([w["w_gate_up"][:, F:], w["w_gate_up"][:, :F]], dim=1)
    ours = fp64.forward(fp64.ModelWeights(CFG, {k: synth.bf16_bits(v) for k, v in bad.items()}), tokens)
    with torch.no_grad():
        lib = _library_model(w)(torch.tensor([tokens])).logits[0].numpy()
    assert np.abs(ours - lib).max() > 1e-2


def test_oracle_attention_matches_torch_sdpa():
    """Causal GQA attention of a prefill chunk (queries at positions 37..63
    over keys 0..63, Hq 8 / Hkv 2) against torch's float64
    scaled_dot_product_attention with the same inclusive causal mask and the
    same contiguous head grouping."""
    rng = np.random.default_rng(5)
    L, n, hq, hkv, d = 64, 27, 8, 2, 128
    q = rng.standard_normal((n, hq, d))
    k = rng.standard_normal((L, hkv, d))
    v = rng.standard_normal((L, hkv, d))
    pos = np.arange(L - n, L)
    scale = 1.0 / np.sqrt(d)
    ours, _ = fp64.attention(q, k, v, pos, scale)
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                  # [1, Hq, n, d]
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)[None]
    mask = torch.from_numpy(np.arange(L)[None, :] <= pos[:, None])     # [n, L], True = attend
    lib = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    lib = lib[0].permute(1, 0, 2).numpy()
    assert np.abs(ours - lib).max() <= 1e-12


def test_oracle_rmsnorm_matches_torch():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((9, 256)) * rng.uniform(0.01, 100, size=(9, 1))
    g = rng.uniform(0.5, 1.5, size=256)
    lib = torch.nn.functional.rms_norm(torch.from_numpy(x), (256,), torch.from_numpy(g), eps=1e-6).numpy()
    assert np.abs(fp64.rmsnorm(x, g, 1e-6) - lib).max() <= 1e-12 * np.abs(lib).max()
