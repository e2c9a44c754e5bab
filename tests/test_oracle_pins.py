"""Pins of the CPU oracle against things other than itself: values printed by
the pages, closed forms, exact rational arithmetic, brute force and algebraic
identities. No GPU; no CUDA library involved.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, a transposed operand, a wrong pairing or mask) fails it.
"""
import itertools
import json
import math
import os
import random
from decimal import Context, Decimal
from fractions import Fraction

import numpy as np
import pytest

from oracle import fp64, ordered

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p2_float_examples.json")


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# "Defeating Nondeterminism in LLM Inference", floating-point non-associativity

def test_associativity_example(golden):
    a = golden["associativity"]
    assert ordered.seq_sum_f64(a["left_grouped"]["terms_in_order"]) == a["left_grouped"]["result"]
    assert ordered.seq_sum_f64(a["right_grouped"]["terms_in_order"]) == a["right_grouped"]["result"]
    # float32 analogue: same loss of the small term
    assert ordered.seq_sum_f32([0.1, 1e20, -1e20]) == 0.0
    assert ordered.seq_sum_f32([1e20, -1e20, 0.1]) == np.float32(0.1)


def _page_shuffle_orders(g):
    """The orders the page's experiment visits: one list shuffled in place
    repeatedly by Python's seeded Mersenne Twister. Returns the values and,
    per position, whether the term is one of the page's int-typed terms."""
    s = g["shuffled_sum"]
    items = [(float(v), i in s["int_terms_initial_order"])
             for i, v in enumerate(s["values_initial_order"])]
    rng = random.Random(s["seed"])
    vals, flags = [], []
    for _ in range(s["shuffles"]):
        rng.shuffle(items)
        vals.append([v for v, _ in items])
        flags.append([f for _, f in items])
    return np.array(vals, dtype=np.float64), np.array(flags, dtype=np.int8)


def test_shuffled_sum_matches_page(golden):
    s = golden["shuffled_sum"]
    vals, flags = _page_shuffle_orders(golden)
    sums = ordered.mixed_sum_rows_f64(vals, flags)
    distinct = sorted(set(sums.tolist()))
    assert len(distinct) == s["distinct_results"]
    assert distinct[0] == s["smallest"]
    assert distinct[1] == s["second_smallest"]
    assert distinct[-1] == s["largest"]
    # the plain left-to-right sum over the same orders: more distinct values,
    # each equal to a Python loop accumulation
    plain = ordered.seq_sum_rows_f64(vals)
    assert len(set(plain.tolist())) == 258
    for row, got in zip(vals[::101], plain[::101]):
        acc = 0.0
        for v in row:
            acc = acc + float(v)
        assert acc == got


def test_all_orders_brute_force():
    """Every order of the 8 values: the exact sum is 0; the oracle's left-to-
    right float64 sum agrees with a plain Python accumulation for each order
    (an implementation that shares nothing with ordered.c)."""
    vals = [1e-10, 1e-5, 1e-2, 1.0, -1e-10, -1e-5, -1e-2, -1.0]
    assert sum(Fraction(v) for v in vals) == 0
    perms = np.array(list(itertools.permutations(vals)), dtype=np.float64)
    sums = ordered.seq_sum_rows_f64(perms)
    for row, got in zip(perms[::97], sums[::97]):
        acc = 0.0
        for v in row:
            acc = acc + float(v)
        assert acc == got
    distinct = np.unique(sums)
    assert len(distinct) == 275
    assert distinct[0] == -2.220446049250313e-16
    assert distinct[-1] == 2.220446049250313e-16


def test_decimal_toy(golden):
    """The page's 3-digit decimal floating-point example, evaluated with the
    decimal module at 3 significant digits (checks the fixture itself)."""
    t = golden["decimal_toy"]
    ctx = Context(prec=t["digits"])
    for a, b, want in t["cases"]:
        assert ctx.add(Decimal(str(a)), Decimal(str(b))) == Decimal(str(want))


def test_grouping_changes_fp32_sums():
    """1024 values summed as 4 x 256, 2 x 512 and left to right: different
    float32 results for values of mixed magnitude, identical for small
    integers (every partial sum exact)."""
    rng = np.random.default_rng(7)
    v = (rng.standard_normal(1024) * np.exp(rng.uniform(-12, 12, 1024))).astype(np.float32)
    r = {ordered.grouped_sum_f32(v, 256), ordered.grouped_sum_f32(v, 512),
         ordered.seq_sum_f32(v)}
    assert len(r) >= 2
    ints = rng.integers(-1000, 1000, 1024).astype(np.float32)
    exact = float(ints.astype(np.int64).sum())
    assert ordered.grouped_sum_f32(ints, 256) == exact
    assert ordered.grouped_sum_f32(ints, 512) == exact
    assert ordered.seq_sum_f32(ints) == exact


# ---------------------------------------------------------------------------
# GEMM: brute force against exact rationals

def _bf16_exact_values(rng, shape, emin=-6, emax=6):
    """Random bf16-representable values with bounded exponents, so every
    product and every sum of a few of them is exact in float64."""
    mant = rng.integers(-255, 256, size=shape)          # 8 significant bits
    exp = rng.integers(emin, emax + 1, size=shape)
    return mant.astype(np.float64) * np.exp2(exp.astype(np.float64) - 7)


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (8, 8, 8), (2, 7, 3)])
def test_gemm_exact(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    A = _bf16_exact_values(rng, (M, K))
    W = _bf16_exact_values(rng, (N, K))
    C = fp64.gemm(A, W)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(A[m, k]) * Fraction(W[n, k]) for k in range(K))
            assert Fraction(C[m, n]) == exact
    # a transposed operand would fail for a non-square case
    if N != K:
        with pytest.raises(ValueError):
            np.asarray(A, np.float64) @ np.asarray(W, np.float64)


def test_gemm_f32_sequential_order():
    """ordered.gemm_f32 is fmaf left to right. With bf16 inputs every product
    is exact in float32, so fmaf(a, b, acc) == float32(a*b) + acc: emulate it
    with numpy float32 scalars and compare bit for bit."""
    rng = np.random.default_rng(3)
    A = fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(rng.standard_normal((4, 37)))).astype(np.float32)
    W = fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(rng.standard_normal((5, 37)))).astype(np.float32)
    C = ordered.gemm_f32(A, W)
    for m in range(4):
        for n in range(5):
            acc = np.float32(0.0)
            for k in range(37):
                acc = np.float32(A[m, k] * W[n, k]) + acc
            assert C[m, n] == acc
    ref = fp64.gemm(A, W)
    assert np.max(np.abs(C - ref)) < 1e-4


# ---------------------------------------------------------------------------
# RMSNorm closed forms

def test_rmsnorm_closed_forms():
    D, eps = 512, 1e-6
    gamma = np.linspace(0.5, 1.5, D)
    for c in [1.0, -3.25, 1e-3, 7.0]:
        y = fp64.rmsnorm(np.full((1, D), c), gamma, eps)
        np.testing.assert_allclose(y[0], c / math.sqrt(c * c + eps) * gamma, rtol=1e-14)
        alt = np.where(np.arange(D) % 2 == 0, c, -c)
        y = fp64.rmsnorm(alt[None, :], gamma, eps)
        np.testing.assert_allclose(y[0], alt / math.sqrt(c * c + eps) * gamma, rtol=1e-14)
    # a single spike: mean of squares is a^2 / D
    x = np.zeros((1, D))
    x[0, 17] = 2.0
    y = fp64.rmsnorm(x, np.ones(D), 0.0)
    assert y[0, 17] == pytest.approx(math.sqrt(D))
    assert np.count_nonzero(y) == 1
    # zero row stays zero (eps keeps it finite)
    assert np.all(fp64.rmsnorm(np.zeros((2, D)), gamma, eps) == 0.0)
    # rows are independent: a row's value does not depend on its neighbours
    rng = np.random.default_rng(0)
    X = rng.standard_normal((6, D))
    np.testing.assert_array_equal(fp64.rmsnorm(X, gamma, eps)[3], fp64.rmsnorm(X[3:4], gamma, eps)[0])


def test_rmsnorm_f32_close_to_fp64():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((8, 512)).astype(np.float32)
    g = rng.uniform(0.5, 1.5, 512).astype(np.float32)
    y32 = ordered.rmsnorm_f32(X, g, 1e-6)
    y64 = fp64.rmsnorm(X, g, 1e-6)
    np.testing.assert_allclose(y32, y64, rtol=2e-6, atol=0)


# ---------------------------------------------------------------------------
# softmax / attention closed forms

def test_softmax_closed_forms():
    np.testing.assert_allclose(fp64.softmax(np.full(7, 3.3)), np.full(7, 1 / 7), rtol=1e-15)
    np.testing.assert_allclose(fp64.softmax(np.array([0.0, math.log(2.0)])), [1 / 3, 2 / 3], rtol=1e-15)
    np.testing.assert_allclose(fp64.softmax(np.array([0.0, -np.inf, 0.0])), [0.5, 0.0, 0.5])


def _rand_qkv(rng, n, L, hq, hkv, d=16):
    return (rng.standard_normal((n, hq, d)), rng.standard_normal((L, hkv, d)),
            rng.standard_normal((L, hkv, d)))


def test_attention_identical_keys_mean_of_values():
    rng = np.random.default_rng(2)
    L, hq, hkv, d = 9, 4, 2, 16
    q, _, v = _rand_qkv(rng, L, L, hq, hkv, d)
    k = np.broadcast_to(rng.standard_normal((1, hkv, d)), (L, hkv, d))
    pos = np.arange(L)
    out, _ = fp64.attention(q, k, v, pos, 0.25)
    for i in range(L):
        for h in range(hq):
            np.testing.assert_allclose(out[i, h], v[: i + 1, h // 2].mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attention_dominant_key_and_first_position():
    rng = np.random.default_rng(3)
    L, hq, hkv, d = 6, 2, 1, 8
    q, k, v = _rand_qkv(rng, 1, L, hq, hkv, d)
    # key 4 aligned with both queries and huge: its value row wins
    k[4, 0] = 1e3 * q[0, 0] / np.linalg.norm(q[0, 0])
    q[0, 1] = q[0, 0]
    out, _ = fp64.attention(q, k, v, [5], 1.0)
    np.testing.assert_allclose(out[0, 0], v[4, 0], rtol=1e-12)
    np.testing.assert_allclose(out[0, 1], v[4, 0], rtol=1e-12)
    # the query at position 0 sees only key 0 (inclusive causal mask)
    out0, _ = fp64.attention(q, k, v, [0], 1.0)
    np.testing.assert_array_equal(out0[0, 0], v[0, 0])


def test_attention_gqa_mapping_and_mask():
    """Head h reads kv head h // group: swapping kv heads swaps the outputs
    of the matching q-head groups, and keys past the query are ignored."""
    rng = np.random.default_rng(4)
    L, hq, hkv, d = 12, 8, 2, 16
    q, k, v = _rand_qkv(rng, 3, L, hq, hkv, d)
    pos = [4, 7, 11]
    out, _ = fp64.attention(q, k, v, pos, 0.3)
    out_sw, _ = fp64.attention(q[:, [4, 5, 6, 7, 0, 1, 2, 3]], k[:, ::-1], v[:, ::-1], pos, 0.3)
    np.testing.assert_allclose(out_sw[:, [4, 5, 6, 7, 0, 1, 2, 3]], out, rtol=1e-13)
    k2, v2 = k.copy(), v.copy()
    k2[5:] = rng.standard_normal(k2[5:].shape)
    v2[5:] = 1e6
    out2, _ = fp64.attention(q[:1], k2, v2, [4], 0.3)
    np.testing.assert_allclose(out2[0], out[0], rtol=1e-13, atol=1e-15)


def test_attention_f32_close_to_fp64():
    rng = np.random.default_rng(5)
    q, k, v = _rand_qkv(rng, 5, 40, 4, 2, 32)
    pos = [3, 10, 20, 30, 39]
    o32 = ordered.attention_f32(q, k, v, pos, 0.2)
    o64, _ = fp64.attention(q, k, v, pos, 0.2)
    np.testing.assert_allclose(o32, o64, rtol=1e-4, atol=1e-5)


@pytest.mark.parametrize("split", [1, 3, 8, 16, 64])
def test_split_merge_identity(split):
    """Split reduction + serial merge equals the direct softmax (algebraic
    identity; pins the merge weights w_s = exp(m_s - M))."""
    rng = np.random.default_rng(split)
    L = 37
    q, k, v = _rand_qkv(rng, 6, L, 4, 2, 16)
    q *= 3.0   # spread the scores so a wrong rescale would show
    pos = [0, 5, 15, 16, 30, 36]
    direct, _ = fp64.attention(q, k, v, pos, 0.7)
    merged = fp64.attention_split(q, k, v, pos, 0.7, split)
    np.testing.assert_allclose(merged, direct, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# RoPE and SwiGLU

def test_rope_closed_forms():
    d, theta = 128, 1e4
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 3, d))
    # position 0 is the identity
    np.testing.assert_array_equal(fp64.rope(x[:1], [0], theta), x[:1])
    # unit vector e_i at position p -> cos/sin of p * theta^(-2i/d) at (i, i + d/2)
    for i in [0, 1, 31, 63]:
        e = np.zeros((1, 1, d))
        e[0, 0, i] = 1.0
        p = 37
        y = fp64.rope(e, [p], theta)[0, 0]
        a = p * theta ** (-2.0 * i / d)
        assert y[i] == pytest.approx(math.cos(a), abs=1e-15)
        assert y[i + d // 2] == pytest.approx(math.sin(a), abs=1e-15)
        assert np.count_nonzero(np.abs(y) > 1e-15) <= 2
    # norms of the (i, i + d/2) pairs are kept
    pos = [0, 1, 5, 100, 4095]
    y = fp64.rope(x, pos, theta)
    n_x = x[..., : d // 2] ** 2 + x[..., d // 2:] ** 2
    n_y = y[..., : d // 2] ** 2 + y[..., d // 2:] ** 2
    np.testing.assert_allclose(n_y, n_x, rtol=1e-12)
    # relative position: <rope(q, m), rope(k, n)> depends on m - n only
    q, k = rng.standard_normal((1, 1, d)), rng.standard_normal((1, 1, d))
    d1 = np.sum(fp64.rope(q, [50], theta) * fp64.rope(k, [20], theta))
    d2 = np.sum(fp64.rope(q, [1030], theta) * fp64.rope(k, [1000], theta))
    assert d1 == pytest.approx(d2, rel=1e-10)


def test_swiglu_closed_forms():
    assert fp64.swiglu(np.array([0.0]), np.array([5.0]))[0] == 0.0
    assert fp64.swiglu(np.array([1.0]), np.array([2.0]))[0] == pytest.approx(2.0 / (1.0 + math.exp(-1.0)))
    assert fp64.swiglu(np.array([40.0]), np.array([1.5]))[0] == pytest.approx(60.0)
    assert fp64.swiglu(np.array([-40.0]), np.array([1.5]))[0] == pytest.approx(-40 * 1.5 * math.exp(-40), rel=1e-6)


def test_argmax_ties_lowest_index():
    x = np.array([[1.0, 3.0, 3.0, 2.0], [0.0, 0.0, 0.0, 0.0], [-1.0, -2.0, -1.0, -5.0]])
    np.testing.assert_array_equal(fp64.argmax_first(x), [1, 0, 0])


# ---------------------------------------------------------------------------
# forward: structural pins (end to end: tests/test_oracle_forward_library.py)

def _tiny_cfg(L=2):
    return dict(n_layers=L, d_model=256, n_q_heads=2, n_kv_heads=1, d_ff=96,
                vocab=50, rms_eps=1e-6, rope_theta=1e4)


def _tiny_weights(cfg, seed=0):
    rng = np.random.default_rng(seed)
    L, D, hq, hkv, F, V = (cfg[k] for k in ("n_layers", "d_model", "n_q_heads", "n_kv_heads", "d_ff", "vocab"))
    def b(*shape, std=0.05):
        return fp64.f64_to_bf16_bits(rng.standard_normal(shape) * std)
    arrays = dict(embed=b(V, D, std=1.0), lm_head=b(V, D), final_norm=fp64.f64_to_bf16_bits(np.ones(D)),
                  attn_norm=fp64.f64_to_bf16_bits(np.ones((L, D))), mlp_norm=fp64.f64_to_bf16_bits(np.ones((L, D))),
                  w_qkv=b(L, (hq + 2 * hkv) * 128, D), w_o=b(L, D, hq * 128),
                  w_gate_up=b(L, 2 * F, D), w_down=b(L, D, F))
    return fp64.ModelWeights(cfg, arrays)


def test_forward_causal():
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg)
    toks = [3, 17, 42, 8, 8, 1]
    full = fp64.forward(w, toks)
    prefix = fp64.forward(w, toks[:4])
    np.testing.assert_allclose(full[:4], prefix, rtol=1e-12, atol=1e-12)
    changed = fp64.forward(w, toks[:5] + [9])
    np.testing.assert_allclose(changed[:5], full[:5], rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(changed[5] - full[5])) > 1e-6


def test_forward_identity_blocks():
    """With W_o = 0 and W_down = 0 every block adds zero: logits are the
    final norm of the embedding times the LM head."""
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg)
    w.a["w_o"] = np.zeros_like(w.a["w_o"])
    w.a["w_down"] = np.zeros_like(w.a["w_down"])
    toks = [5, 6, 7]
    E = fp64.bf16_bits_to_f64(w.a["embed"])
    want = fp64.rmsnorm(E[toks], np.ones(cfg["d_model"]), cfg["rms_eps"]) @ fp64.bf16_bits_to_f64(w.a["lm_head"]).T
    np.testing.assert_allclose(fp64.forward(w, toks), want, rtol=1e-12, atol=1e-12)


def test_forward_one_token_closed_form():
    """A one-token sequence: softmax over a single key is 1, so attention
    returns that token's v rows (one per q-head group) and RoPE at position 0
    is the identity; chain the block by hand."""
    cfg = _tiny_cfg(L=1)
    w = _tiny_weights(cfg, seed=1)
    D, F = cfg["d_model"], cfg["d_ff"]
    tok = 11
    x = fp64.bf16_bits_to_f64(w.a["embed"])[tok]
    Wqkv = fp64.bf16_bits_to_f64(w.a["w_qkv"][0])
    h = x / math.sqrt(np.mean(x * x) + cfg["rms_eps"])
    v = Wqkv[3 * 128:4 * 128] @ h                       # the single kv head's v
    attn = np.concatenate([v, v])                        # both q heads read it
    x = x + fp64.bf16_bits_to_f64(w.a["w_o"][0]) @ attn
    h = x / math.sqrt(np.mean(x * x) + cfg["rms_eps"])
    gu = fp64.bf16_bits_to_f64(w.a["w_gate_up"][0]) @ h
    act = gu[:F] / (1 + np.exp(-gu[:F])) * gu[F:]
    x = x + fp64.bf16_bits_to_f64(w.a["w_down"][0]) @ act
    h = x / math.sqrt(np.mean(x * x) + cfg["rms_eps"])
    want = fp64.bf16_bits_to_f64(w.a["lm_head"]) @ h
    np.testing.assert_allclose(fp64.forward(w, [tok])[0], want, rtol=1e-11, atol=1e-12)


def test_forward_depth_cuts():
    """Cutting the model after l layers: depth n_layers is the plain result
    bit for bit, depth 0 is the final norm of the embedding times the LM
    head, and depth l equals the full forward of the model built from the
    first l layers alone."""
    cfg = _tiny_cfg(L=3)
    w = _tiny_weights(cfg, seed=4)
    toks = [1, 9, 33, 2]
    cuts = fp64.forward(w, toks, depths={0, 1, 3})
    assert set(cuts) == {0, 1, 3}
    assert np.array_equal(cuts[3], fp64.forward(w, toks))
    E = fp64.bf16_bits_to_f64(w.a["embed"])
    want0 = fp64.rmsnorm(E[toks], np.ones(cfg["d_model"]), cfg["rms_eps"]) @ fp64.bf16_bits_to_f64(w.a["lm_head"]).T
    np.testing.assert_allclose(cuts[0], want0, rtol=1e-12, atol=1e-12)
    one = fp64.ModelWeights(dict(cfg, n_layers=1), w.a)
    np.testing.assert_allclose(cuts[1], fp64.forward(one, toks), rtol=0, atol=0)


def test_bf16_rounding_helper():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 3.4e38, 1e-40, np.inf])
    bits = fp64.f64_to_bf16_bits(vals)
    back = fp64.bf16_bits_to_f64(bits)
    assert back[0] == 1.0
    assert back[1] == 1.0                     # tie -> even
    assert back[2] == 1.0 + 2 ** -6           # tie -> even (up)
    assert back[3] == -2.5
    assert back[4] == 0.0
    assert np.isinf(back[5])                  # past the largest finite bf16
    assert back[6] == pytest.approx(1e-40, rel=2 ** -6)
    assert np.isinf(back[7])


# ---------------------------------------------------------------------------
# The fixed float32 order of ordered.rmsnorm_f32 and ordered.attention_f32,
# emulated bit for bit: every float32 operation of the C code is redone here
# with exactly one rounding (fmaf exactly, through rational arithmetic; the
# other operations with numpy float32 scalars, which round once; expf through
# the same libm function the C oracle calls). Planted mistakes of order must
# then fail to match, so the pins can tell orders apart.

import ctypes  # noqa: E402

_libm = ctypes.CDLL("libm.so.6")
_libm.expf.restype = ctypes.c_float
_libm.expf.argtypes = [ctypes.c_float]


def _f32_nearest(q: Fraction) -> np.float32:
    """The float32 nearest to the rational q (ties to even)."""
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    q = abs(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1                                       # now 2^e <= q < 2^(e+1)
    quantum = Fraction(2) ** (max(e, -126) - 23)     # 24 significant bits
    n = q / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return np.float32(sign * float(fl * quantum))


def _fma(a, b, c) -> np.float32:
    return _f32_nearest(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def _rmsnorm_row_emulated(x, g, eps, order=None, fused=True, group_r_gamma=False):
    D = len(x)
    ss = np.float32(0.0)
    for j in (range(D) if order is None else order):
        ss = _fma(x[j], x[j], ss) if fused else np.float32(x[j] * x[j]) + ss
    r = np.float32(1.0) / np.sqrt(ss / np.float32(D) + np.float32(eps))
    if group_r_gamma:
        return np.array([x[j] * (r * g[j]) for j in range(D)], dtype=np.float32)
    return np.array([(x[j] * r) * g[j] for j in range(D)], dtype=np.float32)


def test_rmsnorm_f32_order_bitwise():
    """ordered.rmsnorm_f32: ss = fmaf(x_j, x_j, ss) for j = 0 .. D-1, then
    r = 1 / sqrtf(ss / D + eps), y_j = (x_j r) g_j -- equal bit for bit to
    the emulation; a reversed sum, an unfused multiply-add and x (r g) each
    change some outputs."""
    rng = np.random.default_rng(21)
    M, D = 32, 48
    X = (rng.standard_normal((M, D)) * np.exp(rng.uniform(-3, 3, (M, D)))).astype(np.float32)
    g = rng.uniform(0.5, 1.5, D).astype(np.float32)
    eps = 1e-6
    y = ordered.rmsnorm_f32(X, g, eps)
    want = np.stack([_rmsnorm_row_emulated(X[i], g, eps) for i in range(M)])
    assert np.array_equal(y.view(np.uint32), want.view(np.uint32))
    planted = {
        "reversed sum": [_rmsnorm_row_emulated(X[i], g, eps, order=range(D - 1, -1, -1)) for i in range(M)],
        "mul then add": [_rmsnorm_row_emulated(X[i], g, eps, fused=False) for i in range(M)],
        "x (r g)": [_rmsnorm_row_emulated(X[i], g, eps, group_r_gamma=True) for i in range(M)],
    }
    for name, rows in planted.items():
        assert not np.array_equal(np.stack(rows).view(np.uint32), y.view(np.uint32)), name


def _attention_emulated(q, k, v, q_pos, scale, l_order="forward", one_pass=False):
    n, hq, d = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    sc = np.float32(scale)
    out = np.zeros((n, hq, d), np.float32)
    for i in range(n):
        last = int(q_pos[i])
        for h in range(hq):
            gg = h // group
            s = []
            for j in range(last + 1):
                acc = np.float32(0.0)
                for e in range(d):
                    acc = _fma(q[i, h, e], k[j, gg, e], acc)
                s.append(np.float32(acc * sc))
            if one_pass:
                # a running maximum with rescaling (an online softmax): a
                # different order of operations from the two passes
                m, l = np.float32(-np.inf), np.float32(0.0)
                o = [np.float32(0.0)] * d
                for j in range(last + 1):
                    mn = max(m, s[j])
                    a = np.float32(_libm.expf(float(np.float32(m - mn)))) if m != -np.inf else np.float32(0.0)
                    p = np.float32(_libm.expf(float(np.float32(s[j] - mn))))
                    l = np.float32(a * l) + p
                    o = [_fma(p, v[j, gg, e], np.float32(a * o[e])) for e in range(d)]
                    m = mn
            else:
                m = np.float32(-np.inf)
                for j in range(last + 1):
                    if s[j] > m:
                        m = s[j]
                p = [np.float32(_libm.expf(float(np.float32(s[j] - m)))) for j in range(last + 1)]
                l = np.float32(0.0)
                for j in (range(last + 1) if l_order == "forward" else range(last, -1, -1)):
                    l = l + p[j]
                o = [np.float32(0.0)] * d
                for j in range(last + 1):
                    o = [_fma(p[j], v[j, gg, e], o[e]) for e in range(d)]
            out[i, h] = [o[e] / l for e in range(d)]
    return out


def test_attention_f32_order_bitwise():
    """ordered.attention_f32: s_j = fmaf-dot(q, k_j) over d in order, times
    scale; the maximum over all visible keys first; then p_j = expf(s_j - m),
    l += p_j and o += p_j v_j (fmaf) for j = 0 .. p; o / l. Equal bit for bit
    to the emulation; the denominator summed backwards, and a one-pass
    online softmax, each change some outputs."""
    rng = np.random.default_rng(22)
    L, hq, hkv, d = 14, 2, 1, 8
    q = (rng.standard_normal((3, hq, d)) * 2).astype(np.float32)
    k = rng.standard_normal((L, hkv, d)).astype(np.float32)
    v = rng.standard_normal((L, hkv, d)).astype(np.float32)
    pos = [5, 9, 13]
    got = ordered.attention_f32(q, k, v, pos, 0.35)
    want = _attention_emulated(q, k, v, pos, 0.35)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    for kw in ({"l_order": "backward"}, {"one_pass": True}):
        assert not np.array_equal(_attention_emulated(q, k, v, pos, 0.35, **kw).view(np.uint32),
                                  got.view(np.uint32)), kw


# ---------------------------------------------------------------------------
# forward_rounded: the fp64 forward with each activation stored in a narrower
# format (the basis of the bf16 forward's tolerance)

def test_round_to_formats():
    x = np.array([1.0 + 2 ** -9 + 2 ** -20, -3.0e-3, 0.1, 1e-30])
    np.testing.assert_array_equal(fp64.round_to(x, "bf16"), fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(x)))
    np.testing.assert_array_equal(fp64.round_to(x, "f32"), x.astype(np.float32).astype(np.float64))
    np.testing.assert_array_equal(fp64.round_to(x, None), x)
    # hi + lo carries 16 significant bits: error below 2^-16 relative, and
    # exact for a value that already has that many
    y = fp64.round_to(x, "bf16x2")
    assert np.all(np.abs(y - x) <= 2.0 ** -16 * np.abs(x))
    assert fp64.round_to(np.array([1.0 + 2 ** -15]), "bf16x2")[0] == 1.0 + 2 ** -15
    # IEEE half: 11 significant bits, ties to even, overflow past 65504,
    # subnormal quantum 2^-24
    h = fp64.round_to(np.array([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 65504.0, 65520.0, 2.0 ** -25,
                                1.5 * 2.0 ** -24, -2.5]), "f16")
    assert list(h[:4]) == [1.0, 1 + 2.0 ** -9, 65504.0, np.inf]
    assert list(h[4:]) == [0.0, 2.0 ** -23, -2.5]
    bits = np.array([0x3C00, 0xC000, 0x0001, 0x7BFF], dtype=np.uint16)
    np.testing.assert_array_equal(fp64.f16_bits_to_f64(bits), [1.0, -2.0, 2.0 ** -24, 65504.0])


def test_forward_rounded_without_rounding_is_forward():
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg, seed=7)
    toks = [3, 1, 4, 1, 5, 9]
    assert np.array_equal(fp64.forward_rounded(w, toks, None), fp64.forward(w, toks))
    assert np.array_equal(fp64.forward_rounded(w, toks, {}), fp64.forward(w, toks))


def test_forward_rounded_every_point_is_live():
    """Each storage point, rounded alone to bf16, moves the logits (a point
    the function silently skipped would leave them unchanged), and all of
    the bf16 mode together moves them by about the quadrature sum of the
    single points' errors (independent roundings add in quadrature)."""
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg, seed=8)
    toks = [7, 2, 40, 11, 2, 33, 19, 5]
    ref = fp64.forward(w, toks)
    sq = 0.0
    for point in fp64.ROUNDING["bf16"]:
        err = fp64.forward_rounded(w, toks, {point: "bf16"}) - ref
        assert np.max(np.abs(err)) > 0, point
        sq += np.sum(err ** 2)
    all_err = fp64.forward_rounded(w, toks, dict.fromkeys(fp64.ROUNDING["bf16"], "bf16")) - ref
    ratio = np.sum(all_err ** 2) / sq
    assert 0.5 < ratio < 2.0, ratio


def test_forward_rounded_modes_order():
    """fp32 activations (hi/lo pairs into the GEMMs) are far closer to fp64
    than bf16 activations; bf16 MLP blocks alone fall in between."""
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg, seed=9)
    toks = list(range(1, 30, 3))
    ref = fp64.forward(w, toks)
    e = {m: np.max(np.abs(fp64.forward_rounded(w, toks, m) - ref)) for m in fp64.ROUNDING}
    assert e["f32"] < e["bf16_mlp"] < e["bf16"]
    assert e["f32"] < 1e-2 * e["bf16"]
