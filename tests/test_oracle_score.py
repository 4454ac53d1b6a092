"""Pins of the oracle's score: log of the geometric retention weight.

Make Each Token Count (DBTrimKV), Methodology 2 and Cache What Lasts
(TRIM-KV), core mechanism 2: the weight of token i at step t is
beta_i^(t-i); the score is its logarithm (t-i)*log(beta_i), taken as one
binary32 multiply.
"""
import math

import numpy as np
import pytest

import oracle


def _rand_inputs(n, seed):
    rng = np.random.default_rng(seed)
    t = rng.integers(1, 1 << 24, size=n).astype(np.int32)
    age = np.minimum(rng.integers(1, 1 << 24, size=n), t).astype(np.int32)
    age = np.maximum(age, 1)
    pos = (t - age).astype(np.int32)
    lb = np.log(rng.uniform(1e-4, 1 - 1e-6, size=n)).astype(np.float32)
    return t, pos, lb


def test_score_is_single_rounding_of_exact_product():
    # (t-i) < 2^24 and a binary32 log-retention multiply exactly in binary64
    # (at most 48 significant bits), so rounding that binary64 product once to
    # binary32 is the correctly rounded binary32 product.
    t, pos, lb = _rand_inputs(20000, 1)
    s, ok = oracle.score(t, pos, lb)
    assert ok.all()
    exact = (t.astype(np.float64) - pos.astype(np.float64)) * lb.astype(np.float64)
    ref = exact.astype(np.float32)
    assert np.array_equal(s.view(np.uint32), ref.view(np.uint32))


def test_score_is_log_of_geometric_weight():
    # s must be log(beta^(t-i)) with beta = exp(log beta): checked against
    # math.pow in binary64 for ages where the power does not underflow.
    rng = np.random.default_rng(2)
    for _ in range(2000):
        t = int(rng.integers(50, 5000))
        pos = int(rng.integers(max(0, t - 40), t))
        beta = float(rng.uniform(0.05, 0.999))
        lb = np.float32(math.log(beta))
        s, ok = oracle.score([t], [pos], [lb])
        assert ok[0]
        want = math.log(math.pow(math.exp(float(lb)), t - pos))
        assert abs(float(s[0]) - want) <= 4e-7 * max(1.0, abs(want))


def test_score_direction_and_age():
    # Older tokens of the same beta < 1 score lower; beta^(t-i) at age 1 is beta.
    s, _ = oracle.score([100, 100, 100], [99, 90, 0], [np.float32(math.log(0.5))] * 3)
    assert s[0] == np.float32(math.log(0.5))
    assert s[0] > s[1] > s[2]


def test_negative_zero_is_positive_zero():
    s, ok = oracle.score([10, 10], [3, 9], [np.float32(-0.0), np.float32(0.0)])
    assert ok.all()
    assert s.view(np.uint32).tolist() == [0, 0]


def test_invalid_inputs_refused():
    nan = np.float32("nan")
    _, ok = oracle.score([10, 10, 10, 1 << 24, 10], [10, 11, 3, 0, 3],
                         [np.float32(-1), np.float32(-1), nan, np.float32(-1), np.float32(-np.inf)])
    # age 0, age -1, NaN, age 2^24 refused; -inf allowed (beta = 0 ranks last)
    assert ok.tolist() == [False, False, False, False, True]


def test_minus_infinity_scores_minus_infinity():
    s, ok = oracle.score([10], [3], [np.float32(-np.inf)])
    assert ok[0] and s[0] == -np.inf


@pytest.mark.parametrize("age", [1, 2, 3, 1 << 23, (1 << 24) - 1])
def test_age_exact_in_float(age):
    s, ok = oracle.score([age], [0], [np.float32(-1.0)])
    assert ok[0] and s[0] == -np.float32(age)
