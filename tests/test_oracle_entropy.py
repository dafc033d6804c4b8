"""Pins of oracle.entropy: closed forms (a uniform support of n tokens has
entropy ln n; a one-token support has 0), a hand-worked row, the library
entropy of the full softmax for identity rows, and invariance of the value
to a shift of the logits."""

import math

import numpy as np
import scipy.special
import scipy.stats

import oracle


def _rows(T, k=0, p=1.0, mu=0.0):
    return {"target": np.zeros(T, np.int64), "temperature": np.ones(T, np.float32),
            "top_k": np.full(T, k, np.int32), "top_p": np.full(T, p, np.float32),
            "min_p": np.full(T, mu, np.float32)}


def test_uniform_support_is_log_n():
    # eight tied maxima and a far tail; top-k = 8 keeps exactly the ties
    s = np.concatenate([np.zeros(8), -50.0 - np.arange(40.0)])[None, :]
    assert abs(oracle.entropy(s, _rows(1, k=8))[0] - math.log(8)) < 1e-14
    # min_p = 1 keeps exactly the tied maxima too
    assert abs(oracle.entropy(s, _rows(1, mu=1.0))[0] - math.log(8)) < 1e-14


def test_single_token_support_is_zero():
    s = np.array([[3.0, 1.0, 0.5, -2.0]])
    assert oracle.entropy(s, _rows(1, k=1))[0] == 0.0
    assert oracle.entropy(s, _rows(1, p=1e-6))[0] == 0.0


def test_hand_worked_top_p_row():
    # weights [4, 2, 1, 1], top_p 0.8 keeps ids {0, 1, 2} (the hand-worked
    # support of the golden cases): p = [4/7, 2/7, 1/7],
    # H = 4/7 ln(7/4) + 2/7 ln(7/2) + 1/7 ln 7 = 0.9556998911125343
    s = np.log(np.array([[4.0, 2.0, 1.0, 1.0]]))
    assert abs(oracle.entropy(s, _rows(1, p=0.8))[0] - 0.9556998911125343) < 1e-14


def test_identity_rows_equal_library_entropy_of_softmax():
    rng = np.random.default_rng(9)
    s = rng.standard_normal((16, 300)) * 2.5
    want = scipy.stats.entropy(scipy.special.softmax(s, axis=1), axis=1)
    np.testing.assert_allclose(oracle.entropy(s, _rows(16)), want, rtol=1e-12, atol=1e-13)


def test_shift_invariance_and_bounds():
    rng = np.random.default_rng(10)
    s = rng.standard_normal((8, 100))
    rows = _rows(8, k=30, p=0.9, mu=0.05)
    h = oracle.entropy(s, rows)
    np.testing.assert_allclose(oracle.entropy(s + 7.25, rows), h, rtol=1e-12, atol=1e-14)
    size = oracle.filter_rows(s, rows)["size"]
    assert (h >= 0).all() and (h <= np.log(size) + 1e-12).all()
