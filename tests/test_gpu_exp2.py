"""The attention softmax's FMA-pipe exponential (exp2_poly_f2) against
exp2 in fp64, through its C-ABI self-test: relative error within the
polynomial's fitted bound over the softmax's whole argument range, exact
powers of two at the integers, and the clamp below -125."""
import numpy as np
import pytest
import torch

from block_sparse_attention_flatten_b200 import nabla

pytestmark = pytest.mark.gpu

# 7.49e-5 is the fitted bound with fp32 Horner steps (fit_exp2_poly.py); the
# exponent insertion is exact, so only the final rounding adds a little.
REL_BOUND = 7.6e-5


def _run(x: np.ndarray) -> np.ndarray:
    xt = torch.from_numpy(x.astype(np.float32)).cuda()
    y = nabla.selftest_exp2_poly(xt)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(5)
    dense = np.linspace(-125.0, 8.0, 2_000_000)
    rand = rng.uniform(-125.0, 8.0, 1_000_000)
    near0 = rng.uniform(-2.0, 0.0, 1_000_000)  # where most probabilities live
    x = np.concatenate([dense, rand, near0]).astype(np.float32)
    y = _run(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < REL_BOUND, rel.max()


def test_integers_and_half_integers():
    x = np.concatenate([np.arange(-125, 9), np.arange(-125, 8) + 0.5]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(0.0))
    y = _run(x)
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(y - ref) / ref).max() < REL_BOUND
    # round-to-nearest reduction: at integers f = 0, so 2^n c0 exactly
    ints = x == np.round(x)
    c0 = np.float32(0.99992811)
    np.testing.assert_array_equal(y[ints], np.float64(c0) * np.exp2(x[ints].astype(np.float64)))


def test_clamp_below_minus_125_stays_tiny_and_positive():
    x = np.array([-125.0, -126.0, -149.0, -1000.0, -3.0e38, -126.5], dtype=np.float32)
    y = _run(x)
    assert np.all(y > 0.0)
    assert np.all(y <= 2.0 ** -124)
    assert np.all(np.isfinite(y))
