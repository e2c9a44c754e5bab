"""RMSNorm folded into the next GEMM's A operand ("Defeating Nondeterminism
in LLM Inference", sections "Batch-invariant RMSNorm" and "Batch-invariant
matmul"): bi_gemm_rmsnorm / bi_gemm_rmsnorm_swiglu give the same bits as
bi_rmsnorm_f32in followed by bi_gemm / bi_gemm_swiglu, both where the norm is
applied inside the GEMM (every CTA pair holds at most one output tile) and
where the normed rows go through the workspace; and the product matches the
fp64 oracle (GEMM tolerance on the normed rows, which are themselves within
the RMSNorm tolerance of the oracle's norm)."""
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


def _inputs(M, K, seed):
    x = dev(synth.normal_bf16((M, K), 1.0, seed).float() * 3.0)        # an fp32 residual stream
    gamma = dev(synth.uniform_bf16((K,), 0.5, 1.5, seed + 1))
    return x, gamma


def _unfused(bi, x, gamma):
    h = torch.empty(x.shape, dtype=torch.bfloat16, device="cuda:0")
    bi.bi_rmsnorm(x, gamma, h, EPS)
    return h


def _ws(bi, M, K):
    return torch.empty(bi.bi_gemm_rmsnorm_workspace_size(M, K), dtype=torch.uint8, device="cuda:0")


# the 7B QKV width (24 tiles at M <= 256, 48 at M = 300: folded; 168 at M =
# 1600: through the workspace), rows on both CTAs of a pair, a last K block
# of 8 columns, and a ragged N
SHAPES = [(1, 6144, 4096), (64, 6144, 4096), (200, 6144, 4096), (300, 6144, 4096), (1600, 6144, 4096),
          (37, 264, 4104), (129, 4096, 4096)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_fold_equals_rmsnorm_then_gemm(bi, M, N, K):
    x, gamma = _inputs(M, K, M + K)
    W = dev(synth.normal_bf16((N, K), 0.02, N + 7))
    ws = _ws(bi, M, K)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda:0")
    bi.bi_device_status(clear=True)
    bi.bi_gemm_rmsnorm(x, gamma, EPS, W, C, ws)
    h = _unfused(bi, x, gamma)
    ref = bi.gemm(h, W)
    torch.cuda.synchronize()
    assert bi.bi_device_status(clear=True) == 0
    assert same_bits(C, ref)
    # fp32 output too
    C32 = torch.empty(M, N, dtype=torch.float32, device="cuda:0")
    bi.bi_gemm_rmsnorm(x, gamma, EPS, W, C32, ws, c_dtype=bi.BI_F32)
    assert same_bits(C32, bi.gemm(h, W, torch.float32))
    # a row alone: the same bits
    C1 = torch.empty(1, N, dtype=torch.bfloat16, device="cuda:0")
    bi.bi_gemm_rmsnorm(x[-1:].contiguous(), gamma, EPS, W, C1, _ws(bi, 1, K))
    assert same_bits(C1[0], C[-1])


@pytest.mark.parametrize("M,F,K", [(64, 2048, 4096), (64, 14336, 4096), (130, 1024, 2048)])
def test_fold_swiglu_equals_rmsnorm_then_gemm_swiglu(bi, M, F, K):
    x, gamma = _inputs(M, K, 3 * M + F)
    W = dev(synth.normal_bf16((2 * F, K), 0.02, F + 9))
    out = torch.empty(M, F, dtype=torch.bfloat16, device="cuda:0")
    bi.bi_gemm_rmsnorm_swiglu(x, gamma, EPS, W, out, _ws(bi, M, K))
    h = _unfused(bi, x, gamma)
    ref = torch.empty(M, F, dtype=torch.bfloat16, device="cuda:0")
    bi.bi_gemm_swiglu(h, W, ref)
    assert same_bits(out, ref)


def test_fold_against_the_oracle(bi):
    """Decode-sized (M = 64) folded QKV projection at the 7B width: the normed
    rows within the RMSNorm tolerance of the oracle's norm, and the product
    within the GEMM tolerance of the fp64 product of those rows."""
    M, N, K = 64, 6144, 4096
    x, gamma = _inputs(M, K, 5)
    W = dev(synth.normal_bf16((N, K), 0.02, 6))
    C = torch.empty(M, N, dtype=torch.float32, device="cuda:0")
    bi.bi_gemm_rmsnorm(x, gamma, EPS, W, C, _ws(bi, M, K), c_dtype=bi.BI_F32)
    h = _unfused(bi, x, gamma)
    check(f64(h), fp64.rmsnorm(f64(x), f64(gamma), EPS), np.zeros((M, K)), 0.0, what="normed rows")
    a, w = f64(h), f64(W)
    check(f64(C), fp64.gemm(a, w), fp64.gemm_reduction_scale(a, w), 1.0 / 16, what="folded gemm")
