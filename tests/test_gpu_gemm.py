"""bi_gemm on the GPU against the fp64 oracle, and bitwise invariance across
batch size, batch position and runs ("Defeating Nondeterminism in LLM
Inference", section "Batch-invariant matmul", and the run-to-run matmul test
of section "Introduction"). Tolerance: per element 2^-7 |y| + 2^-7 R / 16."""
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


def _parity(bi, A, W, out_dtype=torch.bfloat16, what=""):
    C = bi.gemm(dev(A), dev(W), out_dtype)
    a, w = f64(A), f64(W)
    check(f64(C), fp64.gemm(a, w), fp64.gemm_reduction_scale(a, w), KAPPA, what=what)
    return C


def test_config1_rmsnorm_then_gemm(bi):
    """X[64,512] -> RMSNorm -> GEMM with W[512,1024] ~ N(0, 1/512). The
    configuration gives W as [K, N]; it is transposed once to the [N, K]
    layout the kernel takes (a reading: the pages fix no layout)."""
    x = synth.normal_bf16((64, 512), 1.0, 0)
    g = synth.uniform_bf16((512,), 0.5, 1.5, 1000)
    W_kn = synth.normal_bf16((512, 1024), 1.0 / np.sqrt(512), 2)
    W = W_kn.t().contiguous()
    n = bi.rmsnorm(dev(x), dev(g), 1e-6)
    C = _parity(bi, n.cpu(), W, what="config1 gemm")
    for r in range(64):
        Cr = bi.gemm(n[r:r + 1], dev(W))
        assert same_bits(Cr[0], C[r])
    for seed in range(1, 9):
        perm = synth.permutation(64, seed).long()
        Cp = bi.gemm(n[perm.cuda()].contiguous(), dev(W))
        assert same_bits(Cp, C[perm.cuda()])


# M straddles the pair tile's row halves (128 rows per CTA, 256 per pair):
# 129 and 255 leave part of the second CTA's rows live, 256 fills the pair,
# 257 and 383 start a second pair tile
@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (5, 264, 72), (130, 520, 200), (257, 1032, 1000),
                                   (128, 256, 64), (300, 776, 4104), (2, 16, 4096), (129, 136, 64),
                                   (255, 384, 136), (256, 128, 520), (383, 264, 264)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_ragged_shapes(bi, M, N, K, out):
    A = synth.normal_bf16((M, K), 1.0, M * 7 + K)
    W = synth.normal_bf16((N, K), 0.02, N * 3 + K)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    C = _parity(bi, A, W, dt, what=f"gemm {M}x{N}x{K} {out}")
    C1 = bi.gemm(dev(A[-1:]), dev(W), dt)
    assert same_bits(C1[0], C[-1])


def test_k_zero_writes_zeros(bi):
    A = torch.ones(3, 8, dtype=torch.bfloat16, device="cuda:0")
    W = torch.ones(16, 8, dtype=torch.bfloat16, device="cuda:0")
    C = torch.full((3, 16), 7.0, dtype=torch.float32, device="cuda:0")
    st = bi.lib.bi_gemm(A.data_ptr(), 8, W.data_ptr(), 8, C.data_ptr(), 16, bi.BI_F32, 3, 16, 0,
                        torch.cuda.current_stream().cuda_stream)
    assert st == bi.BI_OK
    assert torch.all(C == 0)


def test_strided_operands(bi):
    """Leading dimensions larger than the rows (a slice of a wider buffer)."""
    big = synth.normal_bf16((70, 1024), 1.0, 11)
    A = dev(big)[:, 128:640]
    W = dev(synth.normal_bf16((264, 512), 0.02, 12))
    Cbig = torch.zeros(70, 512, dtype=torch.bfloat16, device="cuda:0")
    C = Cbig[:, :264]
    bi.bi_gemm(A, W, C)
    a, w = f64(A), f64(W)
    check(f64(C), fp64.gemm(a, w), fp64.gemm_reduction_scale(a, w), KAPPA, what="strided")
    assert torch.all(Cbig[:, 264:] == 0)


@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096)])
def test_mistral_mlp_sweep_invariance(bi, K, N):
    """The Mistral-7B MLP shapes: row r of every M in {1, 2, 4, ..., 4096} is
    bitwise equal to row r at M = 4096; sampled rows match the oracle."""
    gA = torch.Generator("cuda:0").manual_seed(K)
    gW = torch.Generator("cuda:0").manual_seed(N)
    A = torch.randn(4096, K, device="cuda:0", generator=gA).to(torch.bfloat16)
    W = (torch.randn(N, K, device="cuda:0", generator=gW) * 0.02).to(torch.bfloat16)
    C_full = bi.gemm(A, W)
    M = 1
    while M <= 4096:
        C = bi.gemm(A[:M], W)
        assert same_bits(C, C_full[:M]), f"M={M}"
        M *= 2
    rows = [0, 1, 127, 128, 2049, 4095]
    a, w = f64(A[rows]), f64(W)
    check(f64(C_full[rows]), fp64.gemm(a, w), fp64.gemm_reduction_scale(a, w), KAPPA,
          what=f"sweep K={K} N={N}")
    # batch position: reversed rows give reversed outputs
    C_rev = bi.gemm(A[:512].flip(0).contiguous(), W)
    assert same_bits(C_rev, C_full[:512].flip(0))


def test_run_to_run_1000(bi):
    """The page's repeated-matmul check: 2048 x 2048 bf16, 1000 runs, bitwise."""
    g = torch.Generator("cuda:0").manual_seed(0)
    A = torch.randn(2048, 2048, device="cuda:0", generator=g).to(torch.bfloat16)
    B = torch.randn(2048, 2048, device="cuda:0", generator=g).to(torch.bfloat16)
    ref = bi.gemm(A, B)
    for _ in range(1000):
        assert same_bits(bi.gemm(A, B), ref)


def test_linspace_batch_invariance_demo(bi):
    """The page's slice-then-multiply demo (B = 2048, D = 4096, linspace
    inputs): mm(a[:1], b) vs mm(a, b)[:1]. bi_gemm must give a zero
    difference (inputs rounded to bf16, b passed transposed)."""
    Bn, D = 2048, 4096
    a = torch.linspace(-1000, 1000, Bn * D, device="cuda:0").reshape(Bn, D).to(torch.bfloat16)
    b = torch.linspace(-1000, 1000, D * D, device="cuda:0").reshape(D, D).to(torch.bfloat16)
    W = b.t().contiguous()
    out1 = bi.gemm(a[:1].contiguous(), W, torch.float32)
    out2 = bi.gemm(a, W, torch.float32)[:1]
    assert (out1 - out2).abs().max().item() == 0.0
    assert same_bits(out1, out2)


@pytest.mark.parametrize("M,N,K", [(1, 8, 8192), (5, 264, 8200), (130, 520, 8192), (300, 776, 9000),
                                   (129, 4096, 14336)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_long_k_shapes(bi, M, N, K, out):
    """Narrow weights with a long K (the down projection's shape class): the
    whole K loop of a tile stays in one CTA pair, in order; parity with the
    oracle on ragged shapes, and the last row alone gives the same bits."""
    A = synth.normal_bf16((M, K), 1.0, M * 17 + K)
    W = synth.normal_bf16((N, K), 0.02, N * 19 + K)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    C = _parity(bi, A, W, dt, what=f"long-K gemm {M}x{N}x{K} {out}")
    C1 = bi.gemm(dev(A[-1:]), dev(W), dt)
    assert same_bits(C1[0], C[-1])


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (130, 520, 200), (257, 1032, 1000), (300, 776, 4104)])
@pytest.mark.parametrize("out", ["f16", "f32"])
def test_f16_gemm_parity_and_rows(bi, M, N, K, out):
    """bi_gemm_f16 (the FP16 variant's GEMM: fp16 A and W, the same pair tile
    and K order): parity with the oracle, and the last row alone gives the
    same bits."""
    A = synth.normal_bf16((M, K), 1.0, M * 29 + K).to(torch.float16)
    W = synth.normal_bf16((N, K), 0.02, N * 31 + K).to(torch.float16)
    dt = torch.float16 if out == "f16" else torch.float32
    C = bi.gemm(dev(A), dev(W), dt)
    a = fp64.f16_bits_to_f64(synth.bf16_bits(A))
    w = fp64.f16_bits_to_f64(synth.bf16_bits(W))
    got = fp64.f16_bits_to_f64(synth.bf16_bits(C.cpu())) if out == "f16" else f64(C)
    check(got, fp64.gemm(a, w), fp64.gemm_reduction_scale(a, w), KAPPA, what=f"f16 gemm {M}x{N}x{K} {out}")
    C1 = bi.gemm(dev(A[-1:]), dev(W), dt)
    assert same_bits(C1[0], C[-1])
