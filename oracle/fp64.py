"""float64 definitions of what the batch-invariant path computes.

Test infrastructure only (see the package docstring). Each function is the
plain definition, with no blocking, fusion or reordering: a reader can check it
by eye against the passage it cites.

Sources (page titles and sections):
  [DN]  "Defeating Nondeterminism in LLM Inference"
        - "Batch-invariant RMSNorm": rms_norm(x, w) = x * rsqrt(mean(x^2)) * w
        - "Batch-invariant matmul": a matmul is pointwise products then a
          reduction over K, per output element
        - "Batch-invariant attention": causal attention per query, reduced
          over the keys; split-KV (FlashDecoding) reduction for decode
        - "When are atomic adds needed?": split (tree) reduction finished by
          a separate serial reduction of the partials
  Readings where the pages are silent are marked READING.
"""
from __future__ import annotations

import numpy as np


# --------------------------------------------------------------------------
# bf16 encoding helpers (pure encoding, no arithmetic of the method)

def bf16_bits_to_f64(bits) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 holding the exact same values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits) -> np.ndarray:
    """uint16 IEEE half bit patterns -> float64 holding the exact same values."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """float64 -> nearest bf16 (round to nearest, ties to even) as uint16.

    Rounds the float64 value directly to 8 significant bits (no detour through
    float32, which could double-round a tie); below the normal range the
    quantum stays 2^-133 (bf16 subnormals); past the largest finite bf16 the
    result is inf.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                                 # x = m 2^e, 0.5 <= |m| < 1
    q = np.ldexp(1.0, np.maximum(e, -125) - 8)         # quantum of 8 significant bits
    with np.errstate(over="ignore", invalid="ignore"):
        r = np.round(x / q) * q                        # np.round: half to even
        f = r.astype(np.float32)                       # exact (or inf past the range)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    return np.where(np.isnan(x), np.uint16(0x7FC0), bits).astype(np.uint16)


# --------------------------------------------------------------------------
# [DN] "Batch-invariant RMSNorm"

def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2, last axis) + eps) * gamma.

    The page's definition has no eps; READING: the configuration's eps is
    added inside the square root.
    """
    x = np.asarray(x, dtype=np.float64)
    gamma = np.asarray(gamma, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gamma


# --------------------------------------------------------------------------
# [DN] "Batch-invariant matmul"

def gemm(A, W) -> np.ndarray:
    """C[m, n] = sum_k A[m, k] * W[n, k]  (C = A W^T, weights in nn.Linear
    layout). A library fp64 matmul is the reduction step."""
    return np.asarray(A, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T


def gemm_reduction_scale(A, W) -> np.ndarray:
    """R[m, n] = sqrt(sum_k (A[m, k] W[n, k])^2): the natural size of the
    terms a cancelling dot product adds up (used by the tolerance rule)."""
    A = np.asarray(A, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    return np.sqrt((A * A) @ (W * W).T)


# --------------------------------------------------------------------------
# softmax and attention, [DN] "Batch-invariant attention"

def softmax(s, axis: int = -1) -> np.ndarray:
    """exp(s - max) / sum(exp(s - max)); entries equal to -inf get 0."""
    s = np.asarray(s, dtype=np.float64)
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def attention(q, k, v, q_pos, scale: float):
    """Causal grouped-query attention for the queries of ONE sequence.

    q [n, Hq, d], k/v [L, Hkv, d], q_pos [n] absolute positions: query i
    attends keys 0..q_pos[i] inclusive (READING: the causal mask includes the
    query's own key). q head h uses kv head h // (Hq / Hkv) (READING:
    contiguous groups). Returns (out [n, Hq, d], probs [n, Hq, L]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, hq, d = q.shape
    L, hkv, _ = k.shape
    group = hq // hkv
    q_pos = np.asarray(q_pos, dtype=np.int64)
    keys = np.arange(L)
    masked = keys[None, :] > q_pos[:, None]            # [n, L]
    out = np.zeros((n, hq, d))
    probs = np.zeros((n, hq, L))
    for h in range(hq):
        g = h // group
        s = (q[:, h, :] @ k[:, g, :].T) * scale          # [n, L]
        s = np.where(masked, -np.inf, s)
        p = softmax(s, axis=-1)
        probs[:, h, :] = p
        out[:, h, :] = p @ v[:, g, :]
    return out, probs


def attention_reduction_scale(probs, v, q_heads_per_kv: int) -> np.ndarray:
    """R[i, h, e] = sqrt(sum_j (p_ij v_je)^2) for the tolerance rule."""
    v = np.asarray(v, dtype=np.float64)
    n, hq, L = probs.shape
    R = np.zeros((n, hq, v.shape[2]))
    for h in range(hq):
        g = h // q_heads_per_kv
        R[:, h, :] = np.sqrt((probs[:, h, :] ** 2) @ (v[:, g, :] ** 2))
    return R


def attention_split(q, k, v, q_pos, scale: float, split: int):
    """The same attention computed as a split reduction over fixed-size key
    ranges followed by a serial merge of the partials in split order
    ([DN] "When are atomic adds needed?" and "Batch-invariant attention";
    READING: split boundaries at absolute multiples of `split`, as the
    FlashDecoding step the page ends on needs a split size that does not
    depend on the batch).

    For query i and split s covering keys [s*split, min((s+1)*split, p+1)):
      m_s = max_j s_ij,  l_s = sum_j exp(s_ij - m_s),  O_s = sum_j exp(s_ij - m_s) v_j
    merged as M = max_s m_s, w_s = exp(m_s - M),
      out = sum_s w_s O_s / sum_s w_s l_s.
    In exact arithmetic this equals attention(); in fp64 it agrees to ~1e-15.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, hq, d = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    out = np.zeros((n, hq, d))
    for i in range(n):
        p = int(q_pos[i])
        n_split = p // split + 1
        for h in range(hq):
            g = h // group
            ms, ls, Os = [], [], []
            for s in range(n_split):
                lo, hi = s * split, min((s + 1) * split, p + 1)
                sc = (k[lo:hi, g, :] @ q[i, h, :]) * scale
                m = np.max(sc)
                e = np.exp(sc - m)
                ms.append(m)
                ls.append(np.sum(e))
                Os.append(e @ v[lo:hi, g, :])
            M = max(ms)
            num = np.zeros(d)
            den = 0.0
            for s in range(n_split):
                w = np.exp(ms[s] - M)
                num = num + w * Os[s]
                den = den + w * ls[s]
            out[i, h, :] = num / den
    return out


# --------------------------------------------------------------------------
# pointwise steps ([DN] "How do we make kernels batch-invariant?")

def rope_angles(positions, head_dim: int, theta: float) -> np.ndarray:
    """angle[t, i] = pos_t * theta^(-2 i / head_dim), i < head_dim / 2."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / head_dim)
    return np.outer(np.asarray(positions, dtype=np.float64), inv_freq)


def rope(x, positions, theta: float) -> np.ndarray:
    """Rotary embedding of x [n, H, d] at positions [n].

    READING: rotate-half pairing, element i pairs with element i + d/2:
      y_i = x_i cos a_i - x_{i+d/2} sin a_i,  y_{i+d/2} = x_{i+d/2} cos a_i + x_i sin a_i.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    a = rope_angles(positions, d, theta)[:, None, :]     # [n, 1, d/2]
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(g) -> np.ndarray:
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))


def swiglu(g, u) -> np.ndarray:
    """silu(g) * u."""
    return silu(g) * np.asarray(u, dtype=np.float64)


def argmax_first(x) -> np.ndarray:
    """Greedy token: index of the largest value per row, lowest index on ties
    (READING: the pages fix no tie-break; the lowest index is order-free)."""
    return np.argmax(np.asarray(x), axis=-1).astype(np.int32)


# --------------------------------------------------------------------------
# dense decoder forward

class ModelWeights:
    """16-bit weights of a dense pre-norm decoder (bf16, or fp16 with
    fmt="f16"), held as uint16 bit patterns (numpy), converted to float64 one
    matrix at a time.

    Arrays (nn.Linear layout [out, in]):
      embed [V, D], attn_norm [L, D], w_qkv [L, (Hq + 2 Hkv) d, D],
      w_o [L, D, Hq d], mlp_norm [L, D], w_gate_up [L, 2F, D],
      w_down [L, D, F], final_norm [D], lm_head [V, D].
    """

    def __init__(self, cfg: dict, arrays: dict, fmt: str = "bf16"):
        self.cfg = cfg
        self.a = arrays
        self.fmt = fmt

    def get(self, name, layer=None) -> np.ndarray:
        arr = self.a[name] if layer is None else self.a[name][layer]
        return f16_bits_to_f64(arr) if self.fmt == "f16" else bf16_bits_to_f64(arr)


def forward(weights: ModelWeights, tokens, depths=None):
    """Logits [n, V] for every position of ONE sequence of token ids.

    With `depths` (a collection of layer counts 0 .. n_layers), returns
    instead {l: logits of the model cut after its first l layers}: the final
    RMSNorm and LM head applied to the residual stream after layer l (the
    same loop; depth n_layers is the plain result).

    The block is the pre-norm decoder the configuration names (RMSNorm, RoPE,
    grouped-query causal attention, SwiGLU MLP, untied LM head):
      h = RMSNorm(x);  q, k, v = split(h W_qkv^T);  q, k = RoPE(q), RoPE(k)
      x = x + Attn(q, k, v) W_o^T
      h = RMSNorm(x);  g, u = split(h W_gu^T);  x = x + (silu(g) * u) W_down^T
      logits = RMSNorm_final(x) W_lm^T
    Everything in float64; positions are 0..n-1.
    """
    c = weights.cfg
    D, hq, hkv, dh = c["d_model"], c["n_q_heads"], c["n_kv_heads"], 128
    F = c["d_ff"]
    eps, theta = c["rms_eps"], c["rope_theta"]
    tokens = np.asarray(tokens, dtype=np.int64)
    n = tokens.shape[0]
    pos = np.arange(n)
    scale = 1.0 / np.sqrt(dh)
    x = weights.get("embed")[tokens]                      # [n, D]

    def head(x):
        return gemm(rmsnorm(x, weights.get("final_norm"), eps), weights.get("lm_head"))

    cut = {}
    if depths is not None and 0 in depths:
        cut[0] = head(x)
    for layer in range(c["n_layers"]):
        h = rmsnorm(x, weights.get("attn_norm", layer), eps)
        qkv = gemm(h, weights.get("w_qkv", layer))
        q = qkv[:, : hq * dh].reshape(n, hq, dh)
        k = qkv[:, hq * dh:(hq + hkv) * dh].reshape(n, hkv, dh)
        v = qkv[:, (hq + hkv) * dh:].reshape(n, hkv, dh)
        q = rope(q, pos, theta)
        k = rope(k, pos, theta)
        a, _ = attention(q, k, v, pos, scale)
        x = x + gemm(a.reshape(n, hq * dh), weights.get("w_o", layer))
        h = rmsnorm(x, weights.get("mlp_norm", layer), eps)
        gu = gemm(h, weights.get("w_gate_up", layer))
        x = x + gemm(swiglu(gu[:, :F], gu[:, F:]), weights.get("w_down", layer))
        if depths is not None and layer + 1 in depths:
            cut[layer + 1] = head(x)
    if depths is not None:
        return cut
    return head(x)


# --------------------------------------------------------------------------
# the forward with the storage roundings of a mixed-precision implementation

def round_to(x, kind):
    """x rounded to a storage format, returned in float64.

    kind: None (kept in float64), "f32" (IEEE float32, nearest even),
    "bf16" (bfloat16, nearest even), "f16" (IEEE half, nearest even) or
    "bf16x2" (an fp32 value carried as a pair hi = bf16(v), lo = bf16(v -
    hi), v = f32(x); the value is hi + lo).
    Pure encoding: no arithmetic of the method.
    """
    x = np.asarray(x, dtype=np.float64)
    if kind is None:
        return x
    if kind == "f32":
        return x.astype(np.float32).astype(np.float64)
    if kind == "bf16":
        return bf16_bits_to_f64(f64_to_bf16_bits(x))
    if kind == "f16":
        with np.errstate(over="ignore"):
            return x.astype(np.float16).astype(np.float64)
    if kind == "bf16x2":
        v = x.astype(np.float32).astype(np.float64)
        hi = bf16_bits_to_f64(f64_to_bf16_bits(v))
        lo = bf16_bits_to_f64(f64_to_bf16_bits(v - hi))
        return hi + lo
    raise ValueError(f"unknown storage format {kind!r}")


# Storage format of each activation of the decoder forward, per precision
# mode. The modes are the cross-vendor precision study's variants
# (arXivDaily 2610.05458, abstract): all-bf16 activations, all-fp16
# activations, the full fp32 upcast, and the upcast with only the MLP blocks
# kept in bf16. READING: the
# pages name the variants, not where each rounds; these are the points at
# which a kernel stack stores an activation in a narrower format than fp64:
#   h        RMSNorm output feeding a GEMM (attention block: "h_attn",
#            MLP block: "h_mlp", final: "h_final")
#   qkv      the QKV projection's output
#   qk_rope  q and k after RoPE
#   p        the unnormalised softmax weights exp(s - m) fed to P V (and
#            summed into the softmax denominator)
#   attn     the attention output feeding the O projection
#   gu       gate and up projection outputs; act: silu(g) * u
#   resid    the residual stream after each addition
#   logits   the LM head's output
ROUNDING = {
    "bf16": dict(h_attn="bf16", qkv="bf16", qk_rope="bf16", p="bf16", attn="bf16",
                 h_mlp="bf16", gu="bf16", act="bf16", resid="f32", h_final="bf16", logits="f32"),
    "f16": dict(h_attn="f16", qkv="f16", qk_rope="f16", p="f16", attn="f16",
                h_mlp="f16", gu="f16", act="f16", resid="f32", h_final="f16", logits="f32"),
    "f32": dict(h_attn="bf16x2", qkv="f32", qk_rope="f32", p="f32", attn="bf16x2",
                h_mlp="bf16x2", gu="f32", act="bf16x2", resid="f32", h_final="bf16x2", logits="f32"),
    "bf16_mlp": dict(h_attn="bf16x2", qkv="f32", qk_rope="f32", p="f32", attn="bf16x2",
                     h_mlp="bf16", gu="bf16", act="bf16", resid="f32", h_final="bf16x2", logits="f32"),
}


def attention_rounded(q, k, v, q_pos, scale: float, p_kind):
    """attention() with the softmax weights exp(s - m) rounded to `p_kind`
    before both the weighted sum of the values and the denominator (m the
    row maximum): out = sum_j P_j v_j / sum_j P_j, P_j = round(exp(s_j - m))."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, hq, d = q.shape
    L, hkv, _ = k.shape
    group = hq // hkv
    q_pos = np.asarray(q_pos, dtype=np.int64)
    masked = np.arange(L)[None, :] > q_pos[:, None]
    out = np.zeros((n, hq, d))
    for h in range(hq):
        g = h // group
        s = (q[:, h, :] @ k[:, g, :].T) * scale
        s = np.where(masked, -np.inf, s)
        P = round_to(np.exp(s - np.max(s, axis=-1, keepdims=True)), p_kind)
        out[:, h, :] = (P @ v[:, g, :]) / np.sum(P, axis=-1, keepdims=True)
    return out


def forward_rounded(weights: ModelWeights, tokens, rounding=None):
    """forward() with each activation stored in the format `rounding` names
    (a dict as in ROUNDING, or a mode name; None: every point kept in
    float64, which is forward() itself). Every operation is the float64
    definition; only the stored values are rounded."""
    if isinstance(rounding, str):
        rounding = ROUNDING[rounding]
    r = dict.fromkeys(ROUNDING["bf16"], None)
    if rounding:
        r.update(rounding)
    c = weights.cfg
    D, hq, hkv, dh = c["d_model"], c["n_q_heads"], c["n_kv_heads"], 128
    F = c["d_ff"]
    eps, theta = c["rms_eps"], c["rope_theta"]
    tokens = np.asarray(tokens, dtype=np.int64)
    n = tokens.shape[0]
    pos = np.arange(n)
    scale = 1.0 / np.sqrt(dh)
    x = round_to(weights.get("embed")[tokens], r["resid"])
    for layer in range(c["n_layers"]):
        h = round_to(rmsnorm(x, weights.get("attn_norm", layer), eps), r["h_attn"])
        qkv = round_to(gemm(h, weights.get("w_qkv", layer)), r["qkv"])
        q = qkv[:, : hq * dh].reshape(n, hq, dh)
        k = qkv[:, hq * dh:(hq + hkv) * dh].reshape(n, hkv, dh)
        v = qkv[:, (hq + hkv) * dh:].reshape(n, hkv, dh)
        q = round_to(rope(q, pos, theta), r["qk_rope"])
        k = round_to(rope(k, pos, theta), r["qk_rope"])
        if r["p"] is None:
            a, _ = attention(q, k, v, pos, scale)
        else:
            a = attention_rounded(q, k, v, pos, scale, r["p"])
        a = round_to(a.reshape(n, hq * dh), r["attn"])
        x = round_to(x + gemm(a, weights.get("w_o", layer)), r["resid"])
        h = round_to(rmsnorm(x, weights.get("mlp_norm", layer), eps), r["h_mlp"])
        gu = round_to(gemm(h, weights.get("w_gate_up", layer)), r["gu"])
        act = round_to(swiglu(gu[:, :F], gu[:, F:]), r["act"])
        x = round_to(x + gemm(act, weights.get("w_down", layer)), r["resid"])
    h = round_to(rmsnorm(x, weights.get("final_norm"), eps), r["h_final"])
    return round_to(gemm(h, weights.get("lm_head")), r["logits"])
