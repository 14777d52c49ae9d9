"""Pins for the parity criterion itself: ``oracle.normwise_rel_err``.

Every GPU parity test decides with ||got - ref||_F / ||ref||_F (the normwise relative
error the tolerances are stated in).  These values are worked out by hand, so a wrong
norm (max-abs, L1, squared), a wrong denominator (||got|| or ||got - ref|| + ||ref||) or
swapped arguments fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle


def test_scaled_reference_gives_the_scale_error():
    ref = np.array([[1.0, -2.0, 0.5], [3.0, 0.25, -4.0]])
    for eps in (1e-3, -0.5, 2.0):
        assert oracle.normwise_rel_err(ref * (1 + eps), ref) == pytest.approx(abs(eps), rel=1e-12)


def test_zero_result_is_error_one():
    ref = np.array([1.0, -7.0, 2.5])
    assert oracle.normwise_rel_err(np.zeros(3), ref) == 1.0


def test_both_zero_is_error_zero_and_zero_reference_is_infinite():
    assert oracle.normwise_rel_err(np.zeros((2, 2)), np.zeros((2, 2))) == 0.0
    assert math.isinf(oracle.normwise_rel_err(np.ones(2), np.zeros(2)))


def test_frobenius_norm_not_max_or_l1_or_squared():
    # ref = [[1,2],[2,4]]: ||ref||_F = 5.  got differs by 3 in one entry: error 3/5.
    # (max-abs would give 3/4, L1 3/9, a ratio of squared norms 9/25.)
    ref = np.array([[1.0, 2.0], [2.0, 4.0]])
    got = ref + np.array([[0.0, 0.0], [0.0, 3.0]])
    assert oracle.normwise_rel_err(got, ref) == pytest.approx(0.6, rel=1e-15)
    # spread over several entries: ||(1, -2, 2)|| = 3 -> 3/5 as well
    got2 = ref + np.array([[1.0, -2.0], [2.0, 0.0]])
    assert oracle.normwise_rel_err(got2, ref) == pytest.approx(0.6, rel=1e-15)


def test_denominator_is_the_reference():
    ref = np.array([3.0, 4.0])           # norm 5
    got = 2.0 * ref                      # norm 10, difference norm 5
    assert oracle.normwise_rel_err(got, ref) == pytest.approx(1.0, rel=1e-15)
    assert oracle.normwise_rel_err(ref, got) == pytest.approx(0.5, rel=1e-15)


def test_layout_independent_and_float64():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((7, 5))
    got = ref + 1e-3 * rng.standard_normal((7, 5))
    a = oracle.normwise_rel_err(got, ref)
    assert oracle.normwise_rel_err(got.ravel(), ref.ravel()) == a
    assert oracle.normwise_rel_err(got.T, ref.T) == pytest.approx(a, rel=1e-15)
    # float32 inputs are widened, not compared in float32
    ref32 = np.array([1.0, 1e-8], dtype=np.float32)
    got32 = np.array([1.0, 0.0], dtype=np.float32)
    assert oracle.normwise_rel_err(got32, ref32) == pytest.approx(1e-8, rel=1e-6)
