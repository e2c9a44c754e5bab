"""Paged attention on the GPU: parity with the fp64 oracle, and bitwise
equality of every token's output across decode, chunked prefill (chunks of 1,
64, 512), batch composition and runs ("Defeating Nondeterminism in LLM
Inference", section "Batch-invariant attention": query 1000 must reduce in the
same order with 0 or 999 cached tokens). Tolerance: per element
2^-7 |y| + 2^-7 R with R = sqrt(sum_j (p_j v_j)^2) (kappa = 1 for the bf16
rounding of the softmax weights)."""
import math

import numpy as np
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64
from tests.checker import check
from tests.gpu_common import dev, f64, same_bits

pytestmark = pytest.mark.gpu
D = 128
SCALE = 1.0 / math.sqrt(D)


@pytest.fixture(scope="module")
def bi(cuda_device):
    from invariant_deterministic_03_b200 import bi as mod
    return mod


class Seqs:
    """Per-sequence q/k/v ([L, H, 128] bf16, CPU) and their paged cache."""

    def __init__(self, bi, lens, Hq, Hkv, seed, fill=0.0, spare_pages=3):
        self.lens, self.Hq, self.Hkv = list(lens), Hq, Hkv
        self.q = [synth.normal_bf16((L, Hq, D), 1.0, seed * 1000 + 3 * b) for b, L in enumerate(lens)]
        self.k = [synth.normal_bf16((L, Hkv, D), 1.0, seed * 1000 + 3 * b + 1) for b, L in enumerate(lens)]
        self.v = [synth.normal_bf16((L, Hkv, D), 1.0, seed * 1000 + 3 * b + 2) for b, L in enumerate(lens)]
        self.layout = synth.PagedLayout(lens, seed, spare_pages=spare_pages)
        P = self.layout.num_pages
        self.kc = torch.full((P, Hkv, 16, D), fill, dtype=torch.bfloat16, device="cuda:0")
        self.vc = torch.full((P, Hkv, D, 16), fill, dtype=torch.bfloat16, device="cuda:0")
        for b, L in enumerate(lens):
            slots = self.layout.slots(b, 0, L)
            bi.bi_kv_append(dev(self.k[b].reshape(L, -1)), dev(self.v[b].reshape(L, -1)),
                            dev(slots), self.kc, self.vc)
        self.bt = dev(self.layout.block_table)

    def shape(self, bi, max_kv_len=None):
        return bi.attn_shape(self.Hq, self.Hkv, self.layout.num_pages, self.layout.pages_per_seq,
                             max_kv_len or max(self.lens))

    def oracle(self, b, positions):
        out, probs = fp64.attention(f64(self.q[b][positions]), f64(self.k[b]), f64(self.v[b]),
                                    positions, SCALE)
        R = fp64.attention_reduction_scale(probs, f64(self.v[b]), self.Hq // self.Hkv)
        return out, R


def _decode(bi, S, q_rows, seq_lens, bt, shape):
    B = q_rows.shape[0]
    ws = torch.empty(bi.bi_attn_workspace_size(shape, B), dtype=torch.uint8, device="cuda:0")
    out = torch.empty(B, q_rows.shape[1], dtype=torch.bfloat16, device="cuda:0")
    bi.bi_attn_decode(q_rows, S.kc, S.vc, bt, dev(torch.tensor(seq_lens, dtype=torch.int32)),
                      shape, out, ws)
    return out


def _prefill(bi, S, chunks, shape):
    """chunks: list of (b, start, end) -> one prefill call; returns out rows."""
    q = torch.cat([S.q[b][s:e].reshape(e - s, -1) for b, s, e in chunks])
    cu = [0]
    for _, s, e in chunks:
        cu.append(cu[-1] + e - s)
    seq_lens = [e for _, _, e in chunks]
    bt = S.layout.block_table[[b for b, _, _ in chunks]]
    n = q.shape[0]
    ws = torch.empty(bi.bi_attn_workspace_size(shape, n), dtype=torch.uint8, device="cuda:0")
    out = torch.empty(n, q.shape[1], dtype=torch.bfloat16, device="cuda:0")
    bi.bi_attn_prefill(dev(q), dev(torch.tensor(cu, dtype=torch.int32)), max(e - s for _, s, e in chunks),
                       S.kc, S.vc, dev(bt), dev(torch.tensor(seq_lens, dtype=torch.int32)), shape, out, ws)
    return out


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (16, 8), (64, 8)])
def test_decode_parity(bi, Hq, Hkv):
    lens = [1, 16, 17, 200, 512, 513, 700, 1030]
    S = Seqs(bi, lens, Hq, Hkv, seed=Hq)
    q_rows = torch.stack([S.q[b][L - 1].reshape(-1) for b, L in enumerate(lens)])
    out = _decode(bi, S, dev(q_rows), lens, S.bt, S.shape(bi))
    for b, L in enumerate(lens):
        o64, R = S.oracle(b, [L - 1])
        check(f64(out[b]).reshape(1, Hq, D), o64, R, kappa=1.0, what=f"decode b={b} L={L}")


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (16, 8), (64, 8)])
def test_decode_equals_chunked_prefill(bi, Hq, Hkv):
    """Every token of a 1100-token sequence: decode (one token, its keys
    cached) == prefill in chunks of 1, 64 and 512 == whole prefill, bitwise;
    and each matches the oracle."""
    L = 1100
    S = Seqs(bi, [L], Hq, Hkv, seed=7)
    shape = S.shape(bi)
    # decode of all positions at once: B = L rows sharing one page table
    bt_rep = S.bt.repeat(L, 1)
    q_rows = dev(S.q[0].reshape(L, -1))
    dec = _decode(bi, S, q_rows, list(range(1, L + 1)), bt_rep, shape)
    o64, R = S.oracle(0, list(range(L)))
    check(f64(dec).reshape(L, Hq, D), o64, R, kappa=1.0, what="decode all positions")
    for chunk in [1, 64, 512, L]:
        if chunk == 1:
            starts = list(range(0, L, 97))   # a sample of single-token chunks
        else:
            starts = list(range(0, L, chunk))
        for s0 in starts:
            e0 = min(L, s0 + chunk)
            out = _prefill(bi, S, [(0, s0, e0)], shape)
            assert same_bits(out, dec[s0:e0]), f"chunk {chunk} at {s0}"


def test_workspace_alignment_does_not_change_bits(bi):
    """The split kernel writes its partial rows with 256-bit stores when the
    workspace is 32-byte aligned and 128-bit stores when it is only 16-byte
    aligned; both give the same bits, for decode and prefill."""
    lens = [5, 600, 1300]
    S = Seqs(bi, lens, 32, 8, seed=11)
    shape = S.shape(bi)
    q_rows = dev(torch.stack([S.q[b][L - 1].reshape(-1) for b, L in enumerate(lens)]))
    sl = dev(torch.tensor(lens, dtype=torch.int32))
    n = bi.bi_attn_workspace_size(shape, 1300)
    big = torch.empty(n + 64, dtype=torch.uint8, device="cuda:0")
    assert big.data_ptr() % 32 == 0
    outs = []
    for off in (0, 16):
        ws = big[off:off + n]
        dec = torch.empty(len(lens), q_rows.shape[1], dtype=torch.bfloat16, device="cuda:0")
        bi.bi_attn_decode(q_rows, S.kc, S.vc, S.bt, sl, shape, dec, ws)
        q = dev(S.q[2].reshape(1300, -1))
        pre = torch.empty_like(q)
        bi.bi_attn_prefill(q, dev(torch.tensor([0, 1300], dtype=torch.int32)), 1300, S.kc, S.vc,
                           S.bt[2:3].contiguous(), sl[2:3].contiguous(), shape, pre, ws)
        outs.append((dec, pre))
    assert same_bits(outs[0][0], outs[1][0])
    assert same_bits(outs[0][1], outs[1][1])
    assert same_bits(outs[0][1][-1], outs[0][0][2])     # the last prompt row is the decode row


def test_prefill_bench_workload_sampled(bi):
    """The prefill workload the benchmark times, in the same launch: four
    fresh 2048-token prompts, causal, GQA 32/8, one bi_attn_prefill call.
    Sampled rows (split and tile boundaries, the diagonal, the last row)
    match the fp64 oracle, and each equals, bit for bit, a decode of the same
    position over the same cache."""
    L, B = 2048, 4
    S = Seqs(bi, [L] * B, 32, 8, seed=61)
    shape = S.shape(bi)
    out = _prefill(bi, S, [(b, 0, L) for b in range(B)], shape)
    positions = [0, 127, 128, 511, 512, 1000, 1535, 2047]
    for b in range(B):
        o64, R = S.oracle(b, positions)
        rows = out[b * L + torch.tensor(positions)]
        check(f64(rows).reshape(len(positions), 32, D), o64, R, kappa=1.0, what=f"prefill b={b}")
    # decode of the same positions: one query each, keys up to and including it
    qd = torch.stack([S.q[b][p_].reshape(-1) for b in range(B) for p_ in positions])
    bt = S.bt.repeat_interleave(len(positions), dim=0)
    lens = [p_ + 1 for _ in range(B) for p_ in positions]
    dec = _decode(bi, S, dev(qd), lens, bt, shape)
    idx = torch.tensor([b * L + p_ for b in range(B) for p_ in positions])
    assert same_bits(dec, out[idx])


def test_finishing_pass_work_units_do_not_change_bits(bi):
    """The finishing pass hands a warp units of one token and up to 16 of its
    heads when the call has rows enough, else one row per warp. With 24 q
    heads a 2400-token prefill takes 16-head units, the second one ragged (8
    heads); the same rows from 300-token chunks (one row per warp) are the
    same bits, and sampled rows match the fp64 oracle."""
    L = 2400
    S = Seqs(bi, [L], 24, 6, seed=71)
    shape = S.shape(bi)
    whole = _prefill(bi, S, [(0, 0, L)], shape)
    for s0 in range(0, L, 300):
        part = _prefill(bi, S, [(0, s0, s0 + 300)], shape)
        assert same_bits(part, whole[s0:s0 + 300]), f"chunk at {s0}"
    positions = [0, 511, 512, 1535, 1536, 2047, 2048, 2399]
    o64, R = S.oracle(0, positions)
    check(f64(whole[torch.tensor(positions)]).reshape(len(positions), 24, D), o64, R, kappa=1.0,
          what="prefill 24 heads")


def test_flagged_sequence_inside_work_units(bi):
    """A call large enough for 16-head units in the finishing pass, with one
    sequence whose length exceeds max_kv_len: that sequence's rows are zeros
    and BI_DEV_BAD_SEQLEN is set, and every other row is the same bits as in
    a call without it (8-head units)."""
    L = 600
    S = Seqs(bi, [L] * 4, 32, 8, seed=73)
    shape = S.shape(bi)
    q = dev(torch.cat([S.q[b].reshape(L, -1) for b in range(4)]))
    cu = dev(torch.tensor([0, L, 2 * L, 3 * L, 4 * L], dtype=torch.int32))
    ws = torch.empty(bi.bi_attn_workspace_size(shape, 4 * L), dtype=torch.uint8, device="cuda:0")
    out = torch.empty_like(q)
    bi.bi_device_status(clear=True)
    bi.bi_attn_prefill(q, cu, L, S.kc, S.vc, S.bt, dev(torch.tensor([L, L, 5000, L], dtype=torch.int32)),
                       shape, out, ws)
    torch.cuda.synchronize()
    assert bi.bi_device_status(clear=True) & 0x8      # BI_DEV_BAD_SEQLEN
    assert not out[2 * L:3 * L].float().abs().any()
    good = _prefill(bi, S, [(0, 0, L), (1, 0, L), (3, 0, L)], shape)
    assert bi.bi_device_status(clear=True) == 0
    assert same_bits(out[:2 * L], good[:2 * L])
    assert same_bits(out[3 * L:], good[2 * L:])


def test_batch_composition(bi):
    """A sequence's rows are the same bits alone, co-batched with others of
    mixed lengths and chunk sizes, and at a different batch position."""
    lens = [900, 37, 4100, 513, 64]
    S = Seqs(bi, lens, 32, 8, seed=11)
    shape = S.shape(bi)
    alone = _prefill(bi, S, [(0, 600, 900)], shape)
    mixed = _prefill(bi, S, [(1, 0, 37), (2, 3800, 4100), (0, 600, 900), (3, 512, 513), (4, 0, 64)], shape)
    assert same_bits(mixed[37 + 300:37 + 300 + 300], alone)
    mixed2 = _prefill(bi, S, [(0, 600, 900), (4, 0, 64)], shape)
    assert same_bits(mixed2[:300], alone)
    o64, R = S.oracle(0, list(range(600, 900)))
    check(f64(alone).reshape(300, 32, D), o64, R, kappa=1.0, what="prefill chunk")
    o64, R = S.oracle(2, list(range(3800, 4100)))
    check(f64(mixed[37:337]).reshape(300, 32, D), o64, R, kappa=1.0, what="prefill long")


def test_stale_cache_contents_do_not_leak(bi):
    """Cache slots past a sequence's end hold NaN: outputs are finite and the
    same bits as with a zeroed cache."""
    lens = [5, 300, 1000]
    Sz = Seqs(bi, lens, 32, 8, seed=21, fill=0.0)
    Sn = Seqs(bi, lens, 32, 8, seed=21, fill=float("nan"))
    q_rows = dev(torch.stack([Sz.q[b][L - 1].reshape(-1) for b, L in enumerate(lens)]))
    oz = _decode(bi, Sz, q_rows, lens, Sz.bt, Sz.shape(bi))
    on = _decode(bi, Sn, q_rows, lens, Sn.bt, Sn.shape(bi))
    assert torch.isfinite(on.float()).all()
    assert same_bits(oz, on)
    pz = _prefill(bi, Sz, [(1, 250, 300), (2, 0, 1000)], Sz.shape(bi))
    pn = _prefill(bi, Sn, [(1, 250, 300), (2, 0, 1000)], Sn.shape(bi))
    assert same_bits(pz, pn)


def test_config3_decode(bi):
    """Batch 32, 32/8 GQA heads, head dim 128, lengths uniform in [1, 8192]
    (seed 0), pages from a seeded permutation: every output vs the oracle."""
    lens = synth.attention_lengths(32, 1, 8192, seed=0)
    S = Seqs(bi, lens, 32, 8, seed=0)
    q_rows = dev(torch.stack([S.q[b][L - 1].reshape(-1) for b, L in enumerate(lens)]))
    out = _decode(bi, S, q_rows, lens, S.bt, S.shape(bi, 8192))
    for b, L in enumerate(lens):
        o64, R = S.oracle(b, [L - 1])
        check(f64(out[b]).reshape(1, 32, D), o64, R, kappa=1.0, what=f"config3 b={b} L={L}")
    # run to run
    for _ in range(20):
        assert same_bits(_decode(bi, S, q_rows, lens, S.bt, S.shape(bi, 8192)), out)
    # the max_kv_len bound (grid size, workspace) does not reach the arithmetic
    out2 = _decode(bi, S, q_rows, lens, S.bt, S.shape(bi, 16384))
    assert same_bits(out2, out)


def _logical_k(kc):
    """[P, Hkv, 16, 128] in the blocked core-matrix order -> (slot, d)."""
    P, H = kc.shape[:2]
    return kc.reshape(P, H, 2, 16, 8, 8).permute(0, 1, 2, 4, 3, 5).reshape(P, H, 16, 128)


def _logical_v(vc):
    """[P, Hkv, 128, 16] in the blocked core-matrix order -> (d, slot)."""
    P, H = vc.shape[:2]
    return vc.reshape(P, H, 16, 2, 8, 8).permute(0, 1, 2, 4, 3, 5).reshape(P, H, 128, 16)


def test_kv_append_exact(bi):
    """The cache holds the exact input bytes at the slot's page and offset
    (blocked core-matrix order, see include/bi.h); padding slots are skipped."""
    lens = [40, 3]
    S = Seqs(bi, lens, 32, 8, seed=5)
    K, V = _logical_k(S.kc), _logical_v(S.vc)
    for b, L in enumerate(lens):
        slots = S.layout.slots(b, 0, L).long()
        page, off = slots // 16, slots % 16
        k_got = K[page.cuda(), :, off.cuda(), :]          # [L, Hkv, 128]
        v_got = V[page.cuda(), :, :, off.cuda()]          # [L, Hkv, 128]
        assert same_bits(k_got.cpu(), S.k[b])
        assert same_bits(v_got.cpu(), S.v[b])
    before_k, before_v = S.kc.clone(), S.vc.clone()
    junk = dev(synth.normal_bf16((2, 8 * D), 1.0, 99))
    bi.bi_kv_append(junk, junk, dev(torch.tensor([-1, -5], dtype=torch.int32)), S.kc, S.vc)
    assert same_bits(S.kc, before_k) and same_bits(S.vc, before_v)


def test_bad_page_sets_status(bi):
    """A page id outside the cache is reported through the status word (the
    kernel reads zeros instead and never touches the bad address)."""
    S = Seqs(bi, [40], 32, 8, seed=6)
    bi.bi_device_status(clear=True)
    bt = S.bt.clone()
    bt[0, 1] = S.layout.num_pages + 100
    q_rows = dev(S.q[0][39].reshape(1, -1))
    out = _decode(bi, S, q_rows, [40], bt, S.shape(bi))
    torch.cuda.synchronize()
    st = bi.bi_device_status(clear=True)
    assert st & 0x4
    assert torch.isfinite(out.float()).all()


def test_mixed_batch_decode_then_prefill_subsets(bi):
    """A batch of one-token sequences followed by longer chunks: the decode
    kernel over the leading sequences plus the prefill kernel over the rest
    (cu_q, seq_lens and block table offset to the subset) gives the same bits
    as one prefill call over everything, and a subset call leaves the rows
    it does not cover untouched."""
    lens = [700, 33, 1300, 250, 513]
    S = Seqs(bi, lens, 32, 8, seed=41)
    shape = S.shape(bi)
    chunks = [(0, 699, 700), (1, 32, 33), (2, 1000, 1300), (3, 200, 250), (4, 0, 513)]
    whole = _prefill(bi, S, chunks, shape)
    q = torch.cat([S.q[b][s:e].reshape(e - s, -1) for b, s, e in chunks])
    n = q.shape[0]
    cu = torch.tensor([0, 1, 2, 302, 352, 865], dtype=torch.int32)
    bt = dev(S.layout.block_table[[b for b, _, _ in chunks]])
    sl = dev(torch.tensor([e for _, _, e in chunks], dtype=torch.int32))
    ws = torch.empty(bi.bi_attn_workspace_size(shape, n), dtype=torch.uint8, device="cuda:0")
    out = torch.full((n, q.shape[1]), 7.0, dtype=torch.bfloat16, device="cuda:0")
    nd = 2
    bi.bi_attn_decode(dev(q), S.kc, S.vc, bt, sl[:nd], shape, out[:nd], ws)
    marker = out[:nd].clone()
    max_q = max(e - s for _, s, e in chunks[nd:])   # 513: bounds every chunk's rows
    bi.bi_attn_prefill(dev(q), dev(cu[nd:]), max_q, S.kc, S.vc, bt[nd:].contiguous(), sl[nd:].contiguous(),
                       shape, out, ws)
    assert same_bits(out[:nd], marker)               # the subset call left the decode rows alone
    assert same_bits(out, whole)
    assert bi.bi_device_status(clear=True) == 0


def test_chunk_longer_than_max_q_len_is_reported(bi):
    """max_q_len sizes the grid on the host; a chunk with more rows than it
    (only visible on the device) sets BI_DEV_BAD_SEQLEN instead of passing
    silently."""
    lens = [513]
    S = Seqs(bi, lens, 32, 8, seed=43)
    shape = S.shape(bi)
    q = dev(S.q[0].reshape(513, -1))
    ws = torch.empty(bi.bi_attn_workspace_size(shape, 513), dtype=torch.uint8, device="cuda:0")
    out = torch.empty_like(q)
    bi.bi_device_status(clear=True)
    bi.bi_attn_prefill(q, dev(torch.tensor([0, 513], dtype=torch.int32)), 512, S.kc, S.vc, S.bt,
                       dev(torch.tensor([513], dtype=torch.int32)), shape, out, ws)
    torch.cuda.synchronize()
    assert bi.bi_device_status(clear=True) & 0x8      # BI_DEV_BAD_SEQLEN
    assert not out[512:].float().abs().any()          # the row past max_q_len rows: zeros
