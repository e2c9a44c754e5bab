"""bi_attn_decode_noalloc: decode attention for callers that cannot allocate
device memory (a host application whose own pool owns all device memory, or a
latency-critical loop that cannot afford cudaMalloc's implicit device
synchronisation). It uses the library's fixed device scratch array instead of
a caller workspace; its output must match bi_attn_decode on the same inputs,
on two calls in a row (the second with other lengths, so stale scratch from
the first call cannot leak into it).

This file is collected last on purpose: it must pass when run alone in a
fresh process and after every other test.
"""
import ctypes
import math

import pytest
import torch

from invariant_deterministic_03_b200 import synth
from tests.checker import check
from tests.gpu_common import f64, same_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bi(cuda_device):
    from invariant_deterministic_03_b200 import bi as mod
    return mod


def _decode_case(bi, lens, seed):
    Hq, Hkv, D = 32, 8, 128
    lay = synth.PagedLayout(lens, seed=seed)
    g = torch.Generator("cuda:0").manual_seed(seed)
    kc = torch.randn(lay.num_pages, Hkv, 16, D, device="cuda:0", generator=g).to(torch.bfloat16)
    vc = torch.randn(lay.num_pages, Hkv, D, 16, device="cuda:0", generator=g).to(torch.bfloat16)
    q = torch.randn(len(lens), Hq * D, device="cuda:0", generator=g).to(torch.bfloat16)
    shape = bi.attn_shape(Hq, Hkv, lay.num_pages, lay.pages_per_seq, 8192)
    return q, kc, vc, lay.block_table.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda:0"), shape


def _with_workspace(bi, q, kc, vc, bt, sl, shape):
    ws = torch.empty(bi.bi_attn_workspace_size(shape, q.shape[0]), dtype=torch.uint8, device="cuda:0")
    out = torch.empty_like(q)
    bi.bi_attn_decode(q, kc, vc, bt, sl, shape, out, ws)
    return out


def _noalloc(bi, q, kc, vc, bt, sl, shape):
    """Through the Python binding (which checks the tensors against the shape
    and calls the C entry point)."""
    out = torch.full_like(q, float("nan"))
    bi.bi_attn_decode_noalloc(q, kc, vc, bt, sl, shape, out)
    return out


def test_noalloc_decode_matches_workspace_decode_twice(bi):
    cases = [synth.attention_lengths(32, 1, 8192, seed=0),     # 32 sequences up to 8192 keys
             [1, 17, 513, 4000, 8192, 300, 2]]                   # fewer, other lengths
    for i, lens in enumerate(cases):
        args = _decode_case(bi, lens, seed=40 + i)
        ref = _with_workspace(bi, *args)
        got = _noalloc(bi, *args)
        torch.cuda.synchronize()
        check(f64(got), f64(ref), what=f"noalloc call {i + 1}")
        assert same_bits(got, ref)
    assert bi.bi_device_status(clear=True) == 0


def test_noalloc_binding_rejects_mismatched_tensors(bi):
    """The binding refuses tensors that disagree with the shape fields the
    kernel trusts, before anything reaches the device."""
    q, kc, vc, bt, sl, shape = _decode_case(bi, [5, 6], seed=51)
    out = torch.empty_like(q)
    with pytest.raises(ValueError):
        bi.bi_attn_decode_noalloc(q[:1], kc, vc, bt, sl, shape, out)          # fewer q rows than B
    with pytest.raises(ValueError):
        bi.bi_attn_decode_noalloc(q, kc[:1], vc, bt, sl, shape, out)          # cache below num_pages
    with pytest.raises(ValueError):
        bi.bi_attn_decode_noalloc(q, kc, vc, bt[:1], sl, shape, out)          # block table rows below B


def test_noalloc_rejects_sizes_past_the_scratch(bi):
    q, kc, vc, bt, sl, shape = _decode_case(bi, [5, 6], seed=50)
    big = bi.attn_shape(32, 8, shape.num_pages, shape.max_pages_per_seq, 1 << 20)  # 2048 splits
    out = torch.empty_like(q)
    st = bi.lib.bi_attn_decode_noalloc(q.data_ptr(), q.stride(0), kc.data_ptr(), vc.data_ptr(),
                                       bt.data_ptr(), sl.data_ptr(), 2, ctypes.byref(big),
                                       out.data_ptr(), out.stride(0),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == bi.BI_ERR_WORKSPACE
    assert b"fixed maximum" in bi.lib.bi_last_error()
    need = 2 * 32 * math.ceil((1 << 20) / 512) * 520
    assert need > 16 * 1024 * 1024
