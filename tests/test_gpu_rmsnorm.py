"""bi_rmsnorm on the GPU against the fp64 oracle, and bitwise batch invariance
("Defeating Nondeterminism in LLM Inference", section "Batch-invariant
RMSNorm"). Tolerance: per element 2^-7 relative (kappa = 0: no cancellation)."""
import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64
from tests.checker import check
from tests.gpu_common import dev, f64, same_bits

pytestmark = pytest.mark.gpu
EPS = 1e-6


@pytest.fixture(scope="module")
def bi(cuda_device):
    from invariant_deterministic_03_b200 import bi as mod
    return mod


def _case(M, D, seed):
    x = synth.normal_bf16((M, D), 1.0, seed)
    g = synth.uniform_bf16((D,), 0.5, 1.5, seed + 1000)
    return x, g


def test_config1_parity_and_invariance(bi):
    """X[64, 512] ~ N(0,1), gamma ~ U(0.5, 1.5), eps 1e-6."""
    x, g = _case(64, 512, 0)
    y = bi.rmsnorm(dev(x), dev(g), EPS)
    check(f64(y), fp64.rmsnorm(f64(x), f64(g), EPS), what="rmsnorm 64x512")
    # each row alone, in the full batch, and at 8 seeded random positions
    for r in range(64):
        alone = bi.rmsnorm(dev(x[r:r + 1]), dev(g), EPS)
        assert same_bits(alone[0], y[r])
    for seed in range(1, 9):
        perm = synth.permutation(64, seed).long()
        yp = bi.rmsnorm(dev(x[perm]), dev(g), EPS)
        assert same_bits(yp, y[perm.to(y.device)])


@pytest.mark.parametrize("M,D", [(1, 8), (3, 520), (257, 4096), (5, 4104), (2, 32768), (130, 2048)])
def test_shapes(bi, M, D):
    x, g = _case(M, D, M + D)
    y = bi.rmsnorm(dev(x), dev(g), EPS)
    check(f64(y), fp64.rmsnorm(f64(x), f64(g), EPS), what=f"rmsnorm {M}x{D}")
    y1 = bi.rmsnorm(dev(x[-1:]), dev(g), EPS)
    assert same_bits(y1[0], y[-1])


def test_fp32_input(bi):
    x = torch.randn(33, 4096, generator=synth.gen(5)) * 3.0
    g = synth.uniform_bf16((4096,), 0.5, 1.5, 6)
    y = bi.rmsnorm(dev(x), dev(g), EPS)
    check(f64(y), fp64.rmsnorm(x.double().numpy(), f64(g), EPS), what="rmsnorm fp32-in")
    assert same_bits(bi.rmsnorm(dev(x[7:8]), dev(g), EPS)[0], y[7])


def test_zero_and_constant_rows(bi):
    D = 4096
    x = torch.zeros(4, D, dtype=torch.bfloat16)
    x[1] = 2.5
    x[2, ::2], x[2, 1::2] = 1.5, -1.5
    g = torch.ones(D, dtype=torch.bfloat16)
    y = f64(bi.rmsnorm(dev(x), dev(g), EPS))
    assert np.all(y[0] == 0.0)
    assert np.allclose(y[1], 2.5 / np.sqrt(6.25 + EPS), rtol=2 ** -8)
    assert np.allclose(np.abs(y[2]), 1.5 / np.sqrt(2.25 + EPS), rtol=2 ** -8)


def test_large_batch_sampled(bi):
    """M = 65536, D = 4096: sampled rows against the oracle, and bitwise equal
    to the same rows computed alone."""
    M, D = 65536, 4096
    x = torch.randn(M, D, device="cuda:0", generator=torch.Generator("cuda:0").manual_seed(3)).to(torch.bfloat16)
    g = dev(synth.uniform_bf16((D,), 0.5, 1.5, 4))
    y = bi.rmsnorm(x, g, EPS)
    rows = torch.tensor([0, 1, 4095, 30000, 65535], device="cuda:0")
    check(f64(y[rows]), fp64.rmsnorm(f64(x[rows]), f64(g), EPS), what="rmsnorm sampled")
    ys = bi.rmsnorm(x[rows].contiguous(), g, EPS)
    assert same_bits(ys, y[rows])


def test_run_to_run(bi):
    x, g = _case(64, 512, 9)
    xd, gd = dev(x), dev(g)
    ref = bi.rmsnorm(xd, gd, EPS)
    for _ in range(200):
        assert same_bits(bi.rmsnorm(xd, gd, EPS), ref)
