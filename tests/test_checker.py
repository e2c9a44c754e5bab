"""Negative controls for the tolerance rule: outputs that are wrong in the
ways "GPU program deployment: verifying correctness" describes (an all-zero
output, rows in the wrong place, a single wrong element), and outputs of
plausible kernel mistakes planted in the oracle (an off-by-one causal mask,
the wrong q-to-kv head grouping, a dropped K step), must fail it, and a
correctly rounded output must pass. No GPU."""
import numpy as np
import pytest

from oracle import fp64
from tests.checker import ParityError, check


def _gemm_case(seed=0, M=16, N=24, K=64):
    rng = np.random.default_rng(seed)
    A = fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(rng.standard_normal((M, K))))
    W = fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(rng.standard_normal((N, K)) * 0.02))
    return fp64.gemm(A, W), fp64.gemm_reduction_scale(A, W)


def test_rounded_output_passes():
    y64, R = _gemm_case()
    y = fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(y64))
    check(y, y64, R, kappa=1 / 16, what="bf16-rounded")


def test_all_zero_output_fails():
    y64, R = _gemm_case()
    with pytest.raises(ParityError):
        check(np.zeros_like(y64), y64, R, kappa=1 / 16)


def test_permuted_rows_fail():
    y64, R = _gemm_case()
    with pytest.raises(ParityError):
        check(y64[::-1], y64, R, kappa=1 / 16)


def test_one_element_off_fails():
    y64, R = _gemm_case()
    y = fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(y64))
    i = np.unravel_index(np.argmax(np.abs(y64)), y64.shape)
    y[i] *= 1 + 2.0 ** -5
    with pytest.raises(ParityError):
        check(y, y64, R, kappa=1 / 16)


def test_small_outputs_are_not_swallowed():
    """The page's softmax example: outputs ~2.5e-6, a fixed 0.01 tolerance
    would accept zeros; a relative rule does not."""
    y64 = np.full(4000, 2.5e-6)
    with pytest.raises(ParityError):
        check(np.zeros_like(y64), y64)


def test_nan_and_shape_fail():
    y64, R = _gemm_case()
    y = y64.copy()
    y[0, 0] = np.nan
    with pytest.raises(ParityError):
        check(y, y64, R, kappa=1 / 16)
    with pytest.raises(ParityError):
        check(y64[:, :-1], y64)


def _attention_case(seed=3, L=300, n=40, hq=8, hkv=2, d=128):
    rng = np.random.default_rng(seed)
    r = lambda *s: fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(rng.standard_normal(s)))  # noqa: E731
    q, k, v = r(n, hq, d), r(L, hkv, d), r(L, hkv, d)
    pos = np.arange(L - n, L)
    return q, k, v, pos, 1.0 / np.sqrt(d)


def test_attention_with_an_off_by_one_causal_mask_fails():
    """Each query also seeing the next key (the mask off by one) -- a
    plausible kernel mistake -- must fail the attention tolerance (kappa 1)."""
    q, k, v, pos, scale = _attention_case()
    o64, probs = fp64.attention(q, k, v, pos, scale)
    R = fp64.attention_reduction_scale(probs, v, q.shape[1] // k.shape[1])
    # queries before the last one see one key too many
    wrong, _ = fp64.attention(q[:-1], k, v, pos[:-1] + 1, scale)
    y = o64.copy()
    y[:-1] = wrong
    with pytest.raises(ParityError):
        check(y, o64, R, kappa=1.0)
    # and the correctly masked result, rounded to bf16, passes
    check(fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(o64)), o64, R, kappa=1.0)


def test_attention_with_the_wrong_head_grouping_fails():
    """q head h reading kv head h % Hkv instead of h // (Hq / Hkv)."""
    q, k, v, pos, scale = _attention_case(seed=4)
    hq, hkv = q.shape[1], k.shape[1]
    o64, probs = fp64.attention(q, k, v, pos, scale)
    R = fp64.attention_reduction_scale(probs, v, hq // hkv)
    # the interleaved grouping, expressed through the oracle's contiguous one:
    # head h goes to slot perm[h], which reads kv head perm[h] // G = h % Hkv
    G = hq // hkv
    perm = np.array([(h % hkv) * G + h // hkv for h in range(hq)])
    assert all(perm[h] // G == h % hkv for h in range(hq))
    out, _ = fp64.attention(q[:, np.argsort(perm)], k, v, pos, scale)
    wrong = out[:, perm]
    with pytest.raises(ParityError):
        check(wrong, o64, R, kappa=1.0)


def test_gemm_with_a_dropped_k_step_fails():
    """The last 16-wide K step left out of the reduction (an off-by-one in the
    K loop)."""
    rng = np.random.default_rng(7)
    A = fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(rng.standard_normal((32, 200))))
    W = fp64.bf16_bits_to_f64(fp64.f64_to_bf16_bits(rng.standard_normal((48, 200)) * 0.02))
    y64, R = fp64.gemm(A, W), fp64.gemm_reduction_scale(A, W)
    with pytest.raises(ParityError):
        check(fp64.gemm(A[:, :184], W[:, :184]), y64, R, kappa=1 / 16)
