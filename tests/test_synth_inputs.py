"""The seeded input generators shared by the tests, the bench and the oracle
side (no GPU): reproducible for a seed, different across seeds, and the
paged layout's structure (every page used once, pages of a sequence not
contiguous, slots = page * 16 + offset) holds."""
import torch

from invariant_deterministic_03_b200 import synth


def test_generators_are_seeded():
    a = synth.normal_bf16((33, 65), 1.0, 5)
    assert torch.equal(a.view(torch.int16), synth.normal_bf16((33, 65), 1.0, 5).view(torch.int16))
    assert not torch.equal(a, synth.normal_bf16((33, 65), 1.0, 6))
    assert a.dtype == torch.bfloat16
    u = synth.uniform_bf16((1000,), 0.5, 1.5, 1)
    assert float(u.min()) >= 0.5 and float(u.max()) <= 1.5
    p = synth.permutation(100, 3)
    assert sorted(p.tolist()) == list(range(100)) and torch.equal(p, synth.permutation(100, 3))


def test_paged_layout_structure():
    lens = [1, 16, 17, 300, 777]
    lay = synth.PagedLayout(lens, seed=2, spare_pages=3)
    need = [max(1, -(-L // 16)) for L in lens]
    assert lay.num_pages == sum(need) + 3
    used = [int(p) for b in range(len(lens)) for p in lay.block_table[b, :need[b]]]
    assert len(set(used)) == len(used) == sum(need)          # every page used once
    assert all(0 <= p < lay.num_pages for p in used)
    assert all(int(x) == -1 for b in range(len(lens)) for x in lay.block_table[b, need[b]:])
    pages_777 = lay.block_table[4, :need[4]].tolist()
    assert any(b - a != 1 for a, b in zip(pages_777, pages_777[1:]))  # not one contiguous run
    s = lay.slots(3, 10, 40)
    for i, slot in enumerate(s.tolist()):
        pos = 10 + i
        assert slot == int(lay.block_table[3, pos // 16]) * 16 + pos % 16
