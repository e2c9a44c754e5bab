"""bi_gemm_qkv (the QKV projection with RoPE and the KV-cache write in the
GEMM's epilogue) against the three separate steps it replaces: bi_gemm into
qkv, bi_rope over the q and k heads, bi_kv_append of the k and v heads. The
qkv rows and both whole caches must be the same bits ("Defeating
Nondeterminism in LLM Inference", section "How do we make kernels
batch-invariant?": a pointwise step fused into the producer keeps each
element's arithmetic, and the cache is still written before attention
reads it). Shapes cover the 7B head layout, ragged K, head counts whose
tiles mix q and k heads, a long K, row counts on both CTAs of a pair
tile, padding rows, and bad slots and positions."""
import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from tests.gpu_common import dev, same_bits

pytestmark = pytest.mark.gpu
MAX_POS = 4096


@pytest.fixture(scope="module")
def bi(cuda_device):
    from invariant_deterministic_03_b200 import bi as mod
    return mod


@pytest.fixture(scope="module")
def table(bi):
    cs = torch.empty(MAX_POS * 128, dtype=torch.float32, device="cuda:0")
    bi.bi_rope_table(cs, MAX_POS, 1e4)
    return cs


def _case(bi, table, M, K, Hq, Hkv, seed, slots=None, positions=None, num_pages=64):
    N = (Hq + 2 * Hkv) * 128
    A = dev(synth.normal_bf16((M, K), 1.0, seed))
    W = dev(synth.normal_bf16((N, K), 0.05, seed + 1))
    rng = np.random.default_rng(seed)
    if positions is None:
        positions = rng.integers(0, MAX_POS, size=M)
    if slots is None:
        slots = rng.permutation(num_pages * 16)[:M]
    pos = dev(torch.tensor(np.asarray(positions), dtype=torch.int32))
    sl = dev(torch.tensor(np.asarray(slots), dtype=torch.int32))
    # caches start with the same junk in both runs, so untouched slots compare too
    k0, v0 = bi.new_kv_cache(num_pages, Hkv, "cuda:0", zero=False)
    k0, v0 = k0[0], v0[0]
    k0.copy_(dev(synth.normal_bf16(tuple(k0.shape), 3.0, seed + 2)))
    v0.copy_(dev(synth.normal_bf16(tuple(v0.shape), 3.0, seed + 3)))
    # fused
    qkv1 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda:0")
    kc1, vc1 = k0.clone(), v0.clone()
    bi.bi_device_status(clear=True)
    bi.bi_gemm_qkv(A, W, qkv1, Hq, Hkv, pos, table, MAX_POS, sl, kc1, vc1)
    torch.cuda.synchronize()
    st1 = bi.bi_device_status(clear=True)
    # three steps
    qkv2 = torch.empty_like(qkv1)
    kc2, vc2 = k0.clone(), v0.clone()
    bi.bi_gemm(A, W, qkv2)
    bi.bi_rope(qkv2, Hq + Hkv, pos, table, MAX_POS)
    bi.bi_kv_append(qkv2[:, Hq * 128:(Hq + Hkv) * 128], qkv2[:, (Hq + Hkv) * 128:], sl, kc2, vc2)
    torch.cuda.synchronize()
    st2 = bi.bi_device_status(clear=True)
    assert same_bits(qkv1, qkv2)
    assert same_bits(kc1, kc2)
    assert same_bits(vc1, vc2)
    return st1, st2, qkv1, kc1


# (768, 4096, 32, 8) and (769, 4096, 32, 8): the 7B width on both sides of
# the forward's switch from three launches to the fused one (72 / 96 pair tiles)
@pytest.mark.parametrize("M,K,Hq,Hkv", [(1, 4096, 32, 8), (7, 4096, 32, 8), (130, 4096, 32, 8),
                                        (768, 4096, 32, 8), (769, 4096, 32, 8),
                                        (5, 72, 4, 2), (64, 200, 3, 1), (33, 520, 5, 3),
                                        (17, 8200, 4, 2), (200, 136, 6, 2), (300, 264, 4, 1)])
def test_fused_equals_three_steps(bi, table, M, K, Hq, Hkv):
    st1, st2, _, _ = _case(bi, table, M, K, Hq, Hkv, seed=M * 31 + K)
    assert st1 == 0 and st2 == 0


def test_padding_rows_skip_the_cache(bi, table):
    """slot < 0: the row's q, k, v are still computed and stored in qkv, the
    caches are not touched (both paths)."""
    slots = [5, -1, 17, -1, 200]
    st1, _, _, _ = _case(bi, table, 5, 512, 4, 2, seed=3, slots=slots)
    assert st1 == 0


def test_bad_slot_and_position_set_status(bi, table):
    """A slot past the cache and a position past the RoPE table: the same
    status bits and the same bits in qkv and the caches as the three steps
    (the row stays unrotated, the bad slot is skipped)."""
    st1, st2, _, _ = _case(bi, table, 4, 256, 4, 2, seed=4, slots=[1, 64 * 16 + 3, 9, 30],
                           positions=[3, 7, MAX_POS + 5, 11])
    assert st1 == st2
    assert st1 & 0x2 and st1 & 0x10


def test_row_invariance(bi, table):
    """Row r alone gives the same qkv row and cache slot as in a batch of 96."""
    M, K, Hq, Hkv = 96, 4096, 32, 8
    _, _, qkv, kc = _case(bi, table, M, K, Hq, Hkv, seed=11)
    A = dev(synth.normal_bf16((M, K), 1.0, 11))
    W = dev(synth.normal_bf16(((Hq + 2 * Hkv) * 128, K), 0.05, 12))
    rng = np.random.default_rng(11)
    positions = rng.integers(0, MAX_POS, size=M)
    slots = rng.permutation(64 * 16)[:M]
    for r in (0, 57, 95):
        q1 = torch.empty(1, qkv.shape[1], dtype=torch.bfloat16, device="cuda:0")
        k1, v1 = bi.new_kv_cache(64, Hkv, "cuda:0")
        bi.bi_gemm_qkv(A[r:r + 1], W, q1, Hq, Hkv, dev(torch.tensor([positions[r]], dtype=torch.int32)),
                       table, MAX_POS, dev(torch.tensor([slots[r]], dtype=torch.int32)), k1[0], v1[0])
        assert same_bits(q1[0], qkv[r])
        page, o = divmod(int(slots[r]), 16)
        blk_full = kc[page].flatten(1)   # [Hkv, 2048] blocks of that page
        blk_one = k1[0][page].flatten(1)
        # the row's 8 x 128 keys sit at (o/8)*1024 + (d/8)*64 + (o%8)*8 + d%8 of each block
        d = torch.arange(128, device="cuda:0")
        idx = (o // 8) * 1024 + (d // 8) * 64 + (o % 8) * 8 + d % 8
        assert same_bits(blk_one[:, idx], blk_full[:, idx])
