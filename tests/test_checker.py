"""Negative controls for the tolerance rule: outputs that are wrong in the
ways "GPU program deployment: verifying correctness" describes (an all-zero
output, rows in the wrong place, a single wrong element) must fail it, and a
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
