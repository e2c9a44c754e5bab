"""Host bookkeeping of the forward's paged KV cache (no GPU): page
allocation, prefix sharing between sequences and reference-counted release,
and the batch assembly's slot arithmetic."""
import pytest


@pytest.fixture(scope="module")
def runner():
    # the runner imports the ctypes binding, which wants libbi.so on disk
    # (it is only loaded, never called, here)
    from invariant_deterministic_03_b200 import build
    build.build()
    from invariant_deterministic_03_b200 import runner as mod
    return mod


def _kv(runner, num_pages=32):
    return runner.PagedKV(n_layers=1, num_pages=num_pages, n_kv_heads=1, max_pages_per_seq=16, seed=3,
                          device="cpu")


def test_pages_come_from_a_seeded_permutation(runner):
    a, b = _kv(runner), _kv(runner)
    a.ensure(0, 40)
    b.ensure(0, 40)
    assert a.pages[0] == b.pages[0] and len(a.pages[0]) == 3
    assert len(set(a.pages[0])) == 3
    assert a.slot(0, 17) == a.pages[0][1] * 16 + 1


def test_fork_shares_whole_pages_only(runner):
    kv = _kv(runner)
    kv.ensure(0, 50)
    kv.length[0] = 50
    held = kv.fork(0, 1, 45)                      # 45 tokens: two whole pages
    assert held == 32
    assert kv.pages[1] == kv.pages[0][:2]
    assert kv.length[1] == 32
    assert all(kv.refs[p] == 2 for p in kv.pages[0][:2]) and kv.refs[kv.pages[0][2]] == 1
    kv.ensure(1, 40)                              # the fork's own tail page
    assert kv.pages[1][2] not in kv.pages[0]
    # never more than the source holds
    assert kv.fork(0, 2, 1000) == 48
    with pytest.raises(ValueError):
        kv.fork(0, 1, 16)


def test_release_frees_a_page_when_its_last_holder_goes(runner):
    kv = _kv(runner)
    kv.ensure(0, 64)
    kv.length[0] = 64
    kv.fork(0, 1, 64)
    n_free = len(kv.free)
    kv.release(0)
    assert len(kv.free) == n_free                 # all four pages still held by sequence 1
    kv.release(1)
    assert len(kv.free) == n_free + 4 and not kv.refs


def test_out_of_pages_is_an_error(runner):
    kv = _kv(runner, num_pages=2)
    with pytest.raises(RuntimeError):
        kv.ensure(0, 33)


def test_make_batch_puts_one_token_chunks_first(runner):
    kv = _kv(runner, num_pages=64)
    for seq, n in [(0, 20), (1, 5), (2, 40)]:
        kv.ensure(seq, n)
        kv.length[seq] = n
    toks = list(range(100))
    chunks = [(2, 40, 48), (0, 20, 21), (1, 5, 6)]       # 8 tokens, then two one-token chunks
    b = runner.make_batch(kv, chunks, lambda s: toks, device="cpu")
    assert b["n_decode"] == 2
    assert b["cu_q"].tolist() == [0, 1, 2, 10]           # the one-token chunks are rows 0 and 1
    assert b["positions"].tolist()[:2] == [20, 5]
    assert b["seq_lens"].tolist() == [21, 6, 48]
    assert b["logits_rows"].tolist() == [9, 0, 1]        # logits stay in the order of `chunks`
    b2 = runner.make_batch(kv, chunks, lambda s: toks, device="cpu", decode_first=False)
    assert b2["n_decode"] == 0 and b2["logits_rows"].tolist() == [7, 8, 9]


def test_make_batch_rejects_malformed_steps(runner):
    kv = _kv(runner, num_pages=64)
    kv.ensure(0, 10)
    kv.length[0] = 10
    toks = list(range(100))
    with pytest.raises(ValueError):
        runner.make_batch(kv, [], lambda s: toks, device="cpu")
    with pytest.raises(ValueError):
        runner.make_batch(kv, [(0, 10, 10)], lambda s: toks, device="cpu")       # no tokens
    with pytest.raises(ValueError):
        runner.make_batch(kv, [(0, 10, 11), (0, 11, 12)], lambda s: toks, device="cpu")  # twice
    with pytest.raises(ValueError):
        runner.make_batch(kv, [(0, 9, 11)], lambda s: toks, device="cpu")        # cache holds 10
