"""Seeded synthetic inputs, shared by the tests, the smoke check and the bench.

This module only draws random numbers and builds index structures (page
tables, slot maps, ragged lengths); it holds none of the arithmetic of the
kernels or of the oracle. Everything is generated on the CPU with
``torch.Generator`` seeds, so the same seed gives the same bytes on every host,
and then copied wherever it is needed.

Workload shapes follow the configurations the library is measured on:
RMSNorm then GEMM on a [64, 512] batch, the Mistral-7B MLP GEMM shapes, paged
attention over 32 sequences with GQA 32/8 and lengths uniform in [1, 8192],
and a dense 7B-shaped decoder with random-init weights.
"""
from __future__ import annotations

import math

import torch

PAGE = 16
HEAD_DIM = 128


def gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float = 1.0, seed: int = 0) -> torch.Tensor:
    """N(0, std^2) rounded to bf16 (CPU)."""
    x = torch.randn(*shape, generator=gen(seed), dtype=torch.float32)
    return (x * std).to(torch.bfloat16)


def uniform_bf16(shape, lo: float, hi: float, seed: int = 0) -> torch.Tensor:
    x = torch.rand(*shape, generator=gen(seed), dtype=torch.float32)
    return (lo + (hi - lo) * x).to(torch.bfloat16)


def randint(n, lo: int, hi: int, seed: int) -> torch.Tensor:
    """n integers uniform in [lo, hi] inclusive (int32)."""
    return torch.randint(lo, hi + 1, (n,), generator=gen(seed), dtype=torch.int64).to(torch.int32)


def permutation(n: int, seed: int) -> torch.Tensor:
    return torch.randperm(n, generator=gen(seed)).to(torch.int32)


def bf16_bits(t: torch.Tensor):
    """16-bit (bf16 or fp16) tensor -> numpy uint16 bit patterns (the
    oracle's input form)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


class PagedLayout:
    """A page table for B sequences whose pages come from one seeded random
    permutation of the pool, so consecutive keys of a sequence live in
    non-contiguous pages.

    kv_lens[b] = number of keys of sequence b; pages_per_seq = max pages.
    block_table [B, pages_per_seq] int32 (unused entries -1).
    """

    def __init__(self, kv_lens, seed: int, spare_pages: int = 0):
        self.kv_lens = [int(x) for x in kv_lens]
        self.B = len(self.kv_lens)
        need = [max(1, math.ceil(L / PAGE)) for L in self.kv_lens]
        self.pages_per_seq = max(need) if need else 1
        self.num_pages = sum(need) + spare_pages
        perm = permutation(self.num_pages, seed).tolist()
        bt = torch.full((self.B, self.pages_per_seq), -1, dtype=torch.int32)
        k = 0
        for b in range(self.B):
            for i in range(need[b]):
                bt[b, i] = perm[k]
                k += 1
        self.block_table = bt

    def slots(self, b: int, start: int, count: int) -> torch.Tensor:
        """Cache slots of keys start..start+count-1 of sequence b."""
        pos = torch.arange(start, start + count, dtype=torch.int64)
        page = self.block_table[b].to(torch.int64)[pos // PAGE]
        return (page * PAGE + pos % PAGE).to(torch.int32)


def attention_lengths(B: int, lo: int, hi: int, seed: int):
    """Per-sequence KV lengths uniform in [lo, hi] (the paged-attention
    workload draws 32 of them in [1, 8192])."""
    return randint(B, lo, hi, seed).tolist()


def model_weights(cfg: dict, seed: int, std: float = 0.02) -> dict:
    """Random-init bf16 weights of a dense decoder (nn.Linear layout), norms
    set to one. Each array draws from its own seed (seed*100 + index) so that
    layers can be generated independently."""
    L, D = cfg["n_layers"], cfg["d_model"]
    hq, hkv, F, V = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["d_ff"], cfg["vocab"]
    qkv = (hq + 2 * hkv) * HEAD_DIM
    w = {}
    w["embed"] = normal_bf16((V, D), std, seed * 100 + 1)
    w["lm_head"] = normal_bf16((V, D), std, seed * 100 + 2)
    w["final_norm"] = torch.ones(D, dtype=torch.bfloat16)
    w["attn_norm"] = torch.ones(L, D, dtype=torch.bfloat16)
    w["mlp_norm"] = torch.ones(L, D, dtype=torch.bfloat16)
    w["w_qkv"] = torch.stack([normal_bf16((qkv, D), std, seed * 100 + 10 + 5 * l) for l in range(L)]) if L else torch.empty(0, qkv, D, dtype=torch.bfloat16)
    w["w_o"] = torch.stack([normal_bf16((D, hq * HEAD_DIM), std, seed * 100 + 11 + 5 * l) for l in range(L)]) if L else torch.empty(0, D, hq * HEAD_DIM, dtype=torch.bfloat16)
    w["w_gate_up"] = torch.stack([normal_bf16((2 * F, D), std, seed * 100 + 12 + 5 * l) for l in range(L)]) if L else torch.empty(0, 2 * F, D, dtype=torch.bfloat16)
    w["w_down"] = torch.stack([normal_bf16((D, F), std, seed * 100 + 13 + 5 * l) for l in range(L)]) if L else torch.empty(0, D, F, dtype=torch.bfloat16)
    return w


def to_f16(weights: dict) -> dict:
    """The same weights in fp16 (nearest), for the FP16 precision variant."""
    return {k: v.to(torch.float16) for k, v in weights.items()}
