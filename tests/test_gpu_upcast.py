"""The fp32-activation ("upcast") path on the GPU: bi_gemm_x2, bi_rmsnorm_split,
bi_attn_f32 and bi_forward in the BI_PREC_F32 / BI_PREC_BF16_MLP modes, against
the fp64 oracle, plus bitwise batch invariance in those modes (the
cross-vendor logit-mismatch paper, arXiv 2610.05458 abstract: FP32 upcasting
reduces logit error; keeping the MLP in BF16 keeps most of the gain).

Tolerances follow the arithmetic: a hi/lo bf16 pair carries ~16 significant
bits and the accumulations are fp32, so the per-element rule is the checker's
with 2^-14 in place of 2^-7."""
import math

import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64
from tests.checker import check
from tests.gpu_common import emulated_logit_bounds, dev, f64, same_bits

pytestmark = pytest.mark.gpu
TIGHT = 2.0 ** -14
D = 128


@pytest.fixture(scope="module")
def bi(cuda_device):
    from invariant_deterministic_03_b200 import bi as mod
    return mod


def _split(bi, x32):
    hi = torch.empty(x32.shape, dtype=torch.bfloat16, device=x32.device)
    lo = torch.empty_like(hi)
    bi.bi_split_bf16x2(x32, hi, lo)
    return hi, lo


def _x2_kappa(K: int) -> float:
    """The checker's kappa for the hi/lo GEMM at rel = 2^-14: the tensor
    core accumulates 2 K / 16 K-steps into the fp32 accumulator, each
    rounding toward zero (Fasi, Higham, Mikaitis and Pranesh, "Numerical
    behavior of NVIDIA tensor cores", PeerJ Computer Science 2021), so the
    accumulation error can grow to n_acc * 2^-23 * R; at rel 2^-14 that is
    kappa = n_acc * 2^-9, and never less than 1."""
    n_acc = 2 * ((K + 15) // 16)
    return max(1.0, n_acc * 2.0 ** -9)


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (130, 520, 200), (257, 1032, 4096), (64, 14336, 4096),
                                   (33, 4096, 14336)])
def test_gemm_x2_parity(bi, M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g, dtype=torch.float64).float()
    W = synth.normal_bf16((N, K), 0.02, N + K)
    hi, lo = _split(bi, dev(A))
    C = torch.empty(M, N, dtype=torch.float32, device="cuda:0")
    bi.bi_gemm_x2(hi, lo, dev(W), C)
    a = f64(hi) + f64(lo)
    assert np.max(np.abs(a - A.double().numpy()) / np.maximum(np.abs(A.double().numpy()), 1e-30)) < 2.0 ** -15
    w = f64(W)
    check(f64(C), fp64.gemm(a, w), fp64.gemm_reduction_scale(a, w), kappa=_x2_kappa(K), rel=TIGHT,
          global_rel=TIGHT, what=f"gemm_x2 {M}x{N}x{K}")
    C1 = torch.empty(1, N, dtype=torch.float32, device="cuda:0")
    bi.bi_gemm_x2(hi[-1:].contiguous(), lo[-1:].contiguous(), dev(W), C1)
    assert same_bits(C1[0], C[-1])


def test_rmsnorm_split_parity(bi):
    x = torch.randn(33, 4096, generator=torch.Generator().manual_seed(1)) * 2.0
    gamma = synth.uniform_bf16((4096,), 0.5, 1.5, 2)
    hi = torch.empty(33, 4096, dtype=torch.bfloat16, device="cuda:0")
    lo = torch.empty_like(hi)
    bi.bi_rmsnorm_split(dev(x), dev(gamma), hi, lo, 1e-6)
    check(f64(hi) + f64(lo), fp64.rmsnorm(x.double().numpy(), f64(gamma), 1e-6), rel=TIGHT,
          global_rel=TIGHT, what="rmsnorm_split")
    # the hi part alone is the bf16 RMSNorm of the same fp32 rows
    y = torch.empty_like(hi)
    bi.bi_rmsnorm(dev(x), dev(gamma), y, 1e-6)
    assert same_bits(y, hi)


class F32Seqs:
    def __init__(self, bi, lens, Hq, Hkv, seed):
        self.lens, self.Hq, self.Hkv = list(lens), Hq, Hkv
        g = torch.Generator().manual_seed(seed)
        self.q = [torch.randn(L, Hq, D, generator=g) for L in lens]
        self.k = [torch.randn(L, Hkv, D, generator=g) for L in lens]
        self.v = [torch.randn(L, Hkv, D, generator=g) for L in lens]
        self.layout = synth.PagedLayout(lens, seed)
        P = self.layout.num_pages
        self.kc = torch.full((P, Hkv, 16, D), float("nan"), device="cuda:0")
        self.vc = torch.full((P, Hkv, 16, D), float("nan"), device="cuda:0")
        for b, L in enumerate(lens):
            slots = self.layout.slots(b, 0, L).long()
            page, off = slots // 16, slots % 16
            self.kc[page.cuda(), :, off.cuda(), :] = dev(self.k[b])
            self.vc[page.cuda(), :, off.cuda(), :] = dev(self.v[b])
        self.bt = dev(self.layout.block_table)

    def shape(self, bi):
        return bi.attn_shape(self.Hq, self.Hkv, self.layout.num_pages, self.layout.pages_per_seq,
                             max(self.lens))


def _attn_f32(bi, S, chunks):
    q = torch.cat([S.q[b][s:e].reshape(e - s, -1) for b, s, e in chunks])
    cu = [0]
    for _, s, e in chunks:
        cu.append(cu[-1] + e - s)
    shape = S.shape(bi)
    n = q.shape[0]
    ws = torch.empty(bi.bi_attn_f32_workspace_size(shape, n), dtype=torch.uint8, device="cuda:0")
    out = torch.empty(n, q.shape[1], device="cuda:0")
    bt = dev(S.layout.block_table[[b for b, _, _ in chunks]])
    sl = dev(torch.tensor([e for _, _, e in chunks], dtype=torch.int32))
    bi.bi_attn_f32(dev(q), dev(torch.tensor(cu, dtype=torch.int32)), S.kc, S.vc, bt, sl, shape, out, ws)
    return out


def test_attn_f32_parity_and_invariance(bi):
    lens = [1, 17, 600, 1100]
    S = F32Seqs(bi, lens, 32, 8, seed=3)
    whole = _attn_f32(bi, S, [(b, 0, L) for b, L in enumerate(lens)])
    off = 0
    for b, L in enumerate(lens):
        o64, probs = fp64.attention(S.q[b].double().numpy(), S.k[b].double().numpy(),
                                    S.v[b].double().numpy(), list(range(L)), 1 / math.sqrt(D))
        R = fp64.attention_reduction_scale(probs, S.v[b].double().numpy(), 4)
        check(f64(whole[off:off + L]).reshape(L, 32, D), o64, R, kappa=1.0, rel=TIGHT,
              global_rel=TIGHT, what=f"attn_f32 b={b}")
        off += L
    # chunked prefill and decode give the same bits as the whole prefill
    b, L = 3, 1100
    base = sum(lens[:3])
    for chunk in [1, 64, 512]:
        for s0 in range(0, L, chunk if chunk > 1 else 137):
            e0 = min(L, s0 + chunk)
            got = _attn_f32(bi, S, [(b, s0, e0)])
            assert same_bits(got, whole[base + s0:base + e0]), f"chunk {chunk} at {s0}"


def _engine(cfg, w, seed=0):
    from invariant_deterministic_03_b200 import runner
    wd = {k: v.cuda().contiguous() for k, v in w.items()}
    return runner.Engine(cfg, wd, num_pages=2048, max_pages_per_seq=cfg["max_pos"] // 16,
                         max_tokens=1024, max_logits=64, seed=seed)


MID = dict(n_layers=2, d_model=4096, n_q_heads=32, n_kv_heads=8, d_ff=14336, vocab=32000,
           max_pos=4096, rms_eps=1e-6, rope_theta=1e4)


@pytest.mark.parametrize("precision", ["f32", "bf16_mlp"])
def test_forward_upcast_vs_fp64(bi, precision):
    cfg = dict(MID, precision=precision)
    w = synth.model_weights(cfg, seed=3)
    n = 40
    toks = synth.randint(n, 0, cfg["vocab"] - 1, seed=4).tolist()
    eng = _engine(cfg, w)
    lg = torch.cat([eng.step([(0, p, p + 1)], lambda s: toks)[0] for p in range(n)])
    ow = fp64.ModelWeights(cfg, {k: synth.bf16_bits(v) for k, v in w.items()})
    ref = fp64.forward(ow, toks)
    err = np.abs(f64(lg) - ref)
    if precision == "f32":
        assert err.max() <= 1e-2, f"max abs logit error {err.max():.3e}"
        assert np.linalg.norm(f64(lg) - ref) <= 2.0 ** -8 * np.linalg.norm(ref)
    else:  # MLP activations still bf16: 1.5x the rounding emulation's error
        max_abs, grel, emu = emulated_logit_bounds(ow, toks, "bf16_mlp", ref)
        assert err.max() <= max_abs, f"max abs logit error {err.max():.3e} (emulated {emu['max_abs']:.3e})"
        assert np.linalg.norm(f64(lg) - ref) <= grel * np.linalg.norm(ref)
    # prefill in one chunk gives the same bits as the decode steps
    e2 = _engine(cfg, w, seed=5)
    lg2, _ = e2.step([(0, 0, n)], lambda s: toks)
    assert same_bits(lg2[0], lg[-1])
