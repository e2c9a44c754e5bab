"""A CPU model of the GEMM's fixed-K-split hand-over (no GPU).

When a weight takes the two-way K split, the two CTAs of a cluster each hold
one half-K partial of the tile; each finishes half of the tile's 32-column
chunks (acc0 + acc1) and sends the partner the partials of the other half
through two 16 KB staging slots per direction. Each rank walks eight steps
with the preferred pattern send, send, receive, send, receive, send,
receive, receive, falling back to the other kind when its list of that kind
is exhausted; chunks past N (the ragged last tile) are neither sent nor
finished, by the same test on both ranks.

This model restates that schedule (the step rule and chunk ownership of the
kernel's epilogue in csrc/gemm.cu) and runs both ranks against each other
with the slot limit, for every count of live chunks, checking that no
configuration deadlocks, that each rank receives the chunks it owns in the
order its partner sends them, that every live chunk is finished exactly
once, and, for SwiGLU tiles (gate chunk c paired with up chunk c + 4), that
a rank finishes each up chunk right after its gate chunk, the order its
one-chunk hold relies on.
"""
import pytest

SLOTS = 2           # staging slots per direction
SEND_STEPS = (0, 1, 3, 5)


def owned(rank, i, swiglu):
    """Chunk i (0..3) of the four a rank finishes."""
    return rank * 2 + (i >> 1) + (i & 1) * 4 if swiglu else rank * 4 + i


def schedule(rank, live, swiglu):
    own = [owned(rank, i, swiglu) for i in range(4) if live(owned(rank, i, swiglu))]
    oth = [owned(rank ^ 1, i, swiglu) for i in range(4) if live(owned(rank ^ 1, i, swiglu))]
    seq, n_s, n_r = [], 0, 0
    for step in range(8):
        send = n_s < len(oth) if step in SEND_STEPS else not n_r < len(own)
        if (n_s >= len(oth)) if send else (n_r >= len(own)):
            continue
        if send:
            seq.append(("S", oth[n_s]))
            n_s += 1
        else:
            seq.append(("R", own[n_r]))
            n_r += 1
    return seq, own, oth


def simulate(live, swiglu):
    """Both ranks step whenever they can; returns (finished, per-rank receive
    order) or None on a deadlock."""
    seqs = [schedule(r, live, swiglu)[0] for r in (0, 1)]
    pc, sent, recvd, done = [0, 0], [[], []], [0, 0], [[], []]
    while not all(pc[r] >= len(seqs[r]) for r in (0, 1)):
        progressed = False
        for r in (0, 1):
            if pc[r] >= len(seqs[r]):
                continue
            kind, c = seqs[r][pc[r]]
            peer = r ^ 1
            if kind == "S" and len(sent[r]) - recvd[peer] < SLOTS:
                sent[r].append(c)
                pc[r] += 1
                progressed = True
            elif kind == "R" and len(sent[peer]) > recvd[r]:
                if sent[peer][recvd[r]] != c:
                    raise AssertionError(f"rank {r} expects chunk {c}, slot holds {sent[peer][recvd[r]]}")
                recvd[r] += 1
                done[r].append(c)
                pc[r] += 1
                progressed = True
        if not progressed:
            return None
    return done


def _live(n_live, swiglu):
    # the last tile of a ragged N: chunk c is live while its first column is < N
    return (lambda c: (c & 3) < n_live) if swiglu else (lambda c: c < n_live)


@pytest.mark.parametrize("swiglu,n_live", [(False, n) for n in range(1, 9)] + [(True, n) for n in range(1, 5)])
def test_handover_completes_and_finishes_every_live_chunk_once(swiglu, n_live):
    live = _live(n_live, swiglu)
    done = simulate(live, swiglu)
    assert done is not None, "deadlock"
    finished = sorted(done[0] + done[1])
    assert finished == [c for c in range(8) if live(c)]
    for r in (0, 1):
        _, own, _ = schedule(r, live, swiglu)
        assert done[r] == own          # in the rank's own order
        if swiglu:
            for i, c in enumerate(done[r]):
                if c >= 4:             # an up chunk follows its gate chunk
                    assert i > 0 and done[r][i - 1] == c - 4


def test_one_slot_per_direction_would_deadlock():
    """The schedule needs both slots: with one, the full tile stalls (both
    ranks send twice before their first receive)."""
    global SLOTS
    saved = SLOTS
    try:
        SLOTS = 1
        assert simulate(_live(8, False), False) is None
    finally:
        SLOTS = saved
