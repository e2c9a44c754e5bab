"""The GEMM's fused epilogues against the fp64 oracle and against the
unfused path, bitwise, plus batch invariance ("Defeating Nondeterminism in
LLM Inference", section "Batch-invariant matmul": an epilogue that acts on
one output element after its whole K reduction leaves each element's
reduction order as it was).

* C += A W^T into fp32 (a residual connection): the same bits as an fp32 C
  from bi_gemm followed by one IEEE fp32 addition.
* out = swiglu(A Wg^T, A Wu^T): the same bits as a bf16 bi_gemm of the fused
  [2F, K] weight followed by bi_swiglu. Tolerance against fp64: per element
  2^-7 |y| + 2^-7 R, R = |g u| (bf16 rounding of g, u and the output) plus
  each product's accumulation term R_x / 16 carried through silu(g) u."""
import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64
from tests.checker import check
from tests.gpu_common import dev, f64, same_bits

pytestmark = pytest.mark.gpu
KAPPA = 1.0 / 16


@pytest.fixture(scope="module")
def bi(cuda_device):
    from invariant_deterministic_03_b200 import bi as mod
    return mod


# ragged shapes, rows on both CTAs of a pair tile, and long K on narrow weights
SHAPES = [(1, 8, 8), (5, 264, 72), (130, 520, 200), (300, 776, 4104), (129, 4096, 4096),
          (7, 264, 8200), (130, 4096, 14336), (255, 136, 520), (257, 264, 136)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_add_into_fp32(bi, M, N, K):
    A = synth.normal_bf16((M, K), 1.0, M * 11 + K)
    W = synth.normal_bf16((N, K), 0.02, N * 5 + K)
    C0 = synth.normal_bf16((M, N), 3.0, M + N).float()
    C = dev(C0.clone())
    bi.bi_gemm(dev(A), dev(W), C, add=True)
    # unfused: fp32 product, then one fp32 addition
    P = bi.gemm(dev(A), dev(W), torch.float32)
    assert same_bits(C, dev(C0) + P)
    a, w = f64(A), f64(W)
    check(f64(C), f64(C0) + fp64.gemm(a, w), np.abs(f64(C0)) + fp64.gemm_reduction_scale(a, w), KAPPA,
          what=f"gemm add {M}x{N}x{K}")
    # the last row alone: same bits
    C1 = dev(C0[-1:].clone())
    bi.bi_gemm(dev(A[-1:]), dev(W), C1, add=True)
    assert same_bits(C1[0], C[-1])


def test_gemm_add_k0_leaves_c(bi):
    """K == 0 adds nothing: C keeps its bits."""
    C0 = synth.normal_bf16((4, 16), 1.0, 3).float()
    C = dev(C0.clone())
    buf = torch.zeros(64, dtype=torch.bfloat16, device="cuda:0")   # real pointers for the empty operands
    st = bi.lib.bi_gemm(buf.data_ptr(), 8, buf.data_ptr(), 8, C.data_ptr(), 16, bi.BI_F32_ADD, 4, 16, 0,
                        torch.cuda.current_stream().cuda_stream)
    assert st == bi.BI_OK
    torch.cuda.synchronize()
    assert same_bits(C, dev(C0))


@pytest.mark.parametrize("M,F,K", [(1, 8, 8), (5, 128, 64), (130, 136, 200), (300, 520, 4104),
                                   (64, 1024, 512), (9, 136, 8192), (130, 520, 9000), (200, 136, 136),
                                   (257, 72, 64)])
def test_gemm_swiglu(bi, M, F, K):
    A = synth.normal_bf16((M, K), 1.0, M * 13 + K)
    W = synth.normal_bf16((2 * F, K), 0.05, F * 7 + K)
    out = torch.empty(M, F, dtype=torch.bfloat16, device="cuda:0")
    bi.bi_gemm_swiglu(dev(A), dev(W), out)
    # unfused: bf16 gate/up GEMM, then the SwiGLU kernel
    gu = bi.gemm(dev(A), dev(W))
    ref = torch.empty(M, F, dtype=torch.bfloat16, device="cuda:0")
    bi.bi_swiglu(gu, ref)
    assert same_bits(out, ref)
    a = f64(A)
    wg, wu = f64(W[:F]), f64(W[F:])
    g64, u64 = fp64.gemm(a, wg), fp64.gemm(a, wu)
    # error of silu(g) u: bf16 rounding of g, u and the output (the 2^-7 |g u|
    # and relative terms; |silu'| <= 1.1) plus each product's own fp32
    # accumulation error, bounded as in bi_gemm's rule by R / 16 and carried
    # through silu(g) u: |silu(g)| dU + 1.1 |u| dG
    R = (np.abs(g64 * u64) + (np.abs(fp64.silu(g64)) * fp64.gemm_reduction_scale(a, wu)
                              + 1.1 * np.abs(u64) * fp64.gemm_reduction_scale(a, wg)) / 16)
    check(f64(out), fp64.swiglu(g64, u64), R, 1.0, what=f"gemm swiglu {M}x{F}x{K}")
    # row invariance: the first and last rows alone
    for r in (0, M - 1):
        o1 = torch.empty(1, F, dtype=torch.bfloat16, device="cuda:0")
        bi.bi_gemm_swiglu(dev(A[r:r + 1]), dev(W), o1)
        assert same_bits(o1[0], out[r])
