"""Host-side bookkeeping for bi_forward: page allocation, batch assembly and a
greedy decode loop. Index arithmetic only -- every step of the model runs in
libbi through :class:`invariant_deterministic_03_b200.bi.Model`.

Pages come from a seeded random permutation of the pool, so a sequence's keys
sit in non-contiguous pages, as in a serving engine under load.
"""
from __future__ import annotations

import torch

from . import bi as _bi
from . import synth

PAGE = 16


class PagedKV:
    """KV caches for every layer plus the page tables of live sequences."""

    def __init__(self, n_layers: int, num_pages: int, n_kv_heads: int, max_pages_per_seq: int,
                 seed: int = 0, device="cuda:0", zero=True, precision: int = 0):
        self.num_pages = num_pages
        self.max_pages = max_pages_per_seq
        self.k, self.v = _bi.new_kv_cache(num_pages, n_kv_heads, device, n_layers, zero=zero,
                                          precision=precision)
        self.free = synth.permutation(num_pages, seed).tolist()
        self.pages: dict[int, list[int]] = {}
        self.length: dict[int, int] = {}
        self.refs: dict[int, int] = {}  # page id -> number of sequences whose table holds it

    def ensure(self, seq: int, length: int) -> None:
        pg = self.pages.setdefault(seq, [])
        self.length.setdefault(seq, 0)
        while len(pg) * PAGE < length:
            if not self.free:
                raise RuntimeError("KV cache out of pages")
            if len(pg) >= self.max_pages:
                raise RuntimeError("sequence longer than max_pages_per_seq pages")
            page = self.free.pop(0)
            self.refs[page] = 1
            pg.append(page)

    def slot(self, seq: int, pos: int) -> int:
        return self.pages[seq][pos // PAGE] * PAGE + pos % PAGE

    def release(self, seq: int) -> None:
        for page in self.pages.pop(seq, []):
            self.refs[page] -= 1
            if self.refs[page] == 0:
                del self.refs[page]
                self.free.append(page)
        self.length.pop(seq, None)

    def fork(self, src: int, dst: int, n_tokens: int) -> int:
        """Prefix reuse: `dst` starts with the cached keys of the first
        n_tokens of `src`, by sharing src's whole pages (the same page ids in
        both block tables; nothing is copied). A partly filled last page is
        not shared -- `dst` recomputes those tokens into pages of its own, so
        no sequence ever writes into a page another one reads. Returns the
        number of tokens `dst` now holds (n_tokens rounded down to a page).
        Attention walks tiles and splits at absolute key offsets, so `dst`'s
        outputs are the same bits as if it had computed the prefix itself."""
        if dst in self.pages:
            raise ValueError(f"sequence {dst} already exists")
        n_tokens = min(n_tokens, self.length.get(src, 0))
        shared = self.pages[src][: n_tokens // PAGE]
        for page in shared:
            self.refs[page] += 1
        self.pages[dst] = list(shared)
        self.length[dst] = len(shared) * PAGE
        return self.length[dst]


def make_batch(kv: PagedKV, chunks, tokens_of, device="cuda:0", decode_first: bool = True):
    """chunks: list of (seq, start, end) -- tokens start..end-1 of `seq` are
    processed in this step (their keys are written, then attended). The keys
    0..start-1 must already be cached. Returns the device batch dict for
    Model.forward with one logits row per chunk (its last token), in the order
    of `chunks`. With decode_first, one-token chunks are laid out first and
    counted in n_decode, so their attention runs in the decode kernel (a row's
    bits do not depend on which kernel or which batch position computes it)."""
    if not chunks:
        raise ValueError("empty batch")
    for seq, s, e in chunks:
        if e <= s:
            raise ValueError(f"sequence {seq}: empty chunk {s}..{e}")
    if len({seq for seq, _, _ in chunks}) != len(chunks):
        raise ValueError("a sequence appears twice in one step")
    order = list(range(len(chunks)))
    n_decode = 0
    if decode_first:
        one = [i for i, (_, s, e) in enumerate(chunks) if e - s == 1]
        rest = [i for i, (_, s, e) in enumerate(chunks) if e - s != 1]
        order, n_decode = one + rest, len(one)
    toks, pos, slots, cu, lens = [], [], [], [0], []
    last_row = {}
    for i in order:
        seq, s, e = chunks[i]
        if kv.length.get(seq, 0) != s:
            raise ValueError(f"sequence {seq}: cache holds {kv.length.get(seq, 0)} keys, chunk starts at {s}")
        kv.ensure(seq, e)
        t = tokens_of(seq)
        for p in range(s, e):
            toks.append(int(t[p]))
            pos.append(p)
            slots.append(kv.slot(seq, p))
        cu.append(cu[-1] + e - s)
        lens.append(e)
        last_row[i] = cu[-1] - 1
    rows = [last_row[i] for i in range(len(chunks))]
    bt = torch.full((len(chunks), kv.max_pages), -1, dtype=torch.int32)
    for j, i in enumerate(order):
        pg = kv.pages[chunks[i][0]]
        bt[j, : len(pg)] = torch.tensor(pg, dtype=torch.int32)
    i32 = lambda x: torch.tensor(x, dtype=torch.int32, device=device)  # noqa: E731
    batch = {"tokens": i32(toks), "positions": i32(pos), "slot_mapping": i32(slots),
             "cu_q": i32(cu), "seq_lens": i32(lens), "block_table": bt.to(device),
             "logits_rows": i32(rows), "max_q_len": max(e - s for _, s, e in chunks),
             "max_kv_len": max(lens), "n_decode": n_decode}
    return batch


def commit(kv: PagedKV, chunks) -> None:
    """Record that the chunks' keys are now cached."""
    for seq, _, e in chunks:
        kv.length[seq] = e


class Engine:
    """A model, its caches and one reusable workspace."""

    def __init__(self, cfg: dict, weights_dev: dict, num_pages: int, max_pages_per_seq: int,
                 max_tokens: int, max_logits: int, seed: int = 0, device="cuda:0"):
        self.cfg = cfg
        self.model = _bi.Model(cfg, weights_dev)
        self.kv = PagedKV(cfg["n_layers"], num_pages, cfg["n_kv_heads"], max_pages_per_seq,
                          seed, device, precision=self.model.precision)
        self.device = device
        self.max_tokens, self.max_logits = max_tokens, max_logits
        ws = self.model.workspace_size(max_tokens, max_logits, cfg["max_pos"])
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)

    def step(self, chunks, tokens_of):
        """Runs one forward over the chunks; returns (logits [n_chunks, V]
        fp32, greedy next tokens [n_chunks] int32), both on the device."""
        b = make_batch(self.kv, chunks, tokens_of, self.device)
        if b["tokens"].shape[0] > self.max_tokens or len(chunks) > self.max_logits:
            raise ValueError("batch larger than the workspace")
        b["max_kv_len"] = self.cfg["max_pos"]   # fixed bound: sizes grid and workspace only
        logits = torch.empty(len(chunks), self.cfg["vocab"], dtype=torch.float32, device=self.device)
        nxt = torch.empty(len(chunks), dtype=torch.int32, device=self.device)
        self.model.forward(b, self.kv.k, self.kv.v, logits, nxt, self.ws)
        commit(self.kv, chunks)
        return logits, nxt
