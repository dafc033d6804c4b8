"""Pin of oracle.logprob_on_prefix: at the oracle's own support size it is
the forward's logprob; at another size it is the log-softmax restricted to
that many leading tokens of the order, worked by hand."""

import math

import numpy as np

import oracle


def test_prefix_logprob_equals_forward_at_the_oracle_size():
    rng = np.random.default_rng(3)
    T, V = 20, 50
    s = rng.standard_normal((T, V)) * 2
    rows = {"target": rng.integers(0, V, T), "temperature": np.ones(T, np.float32),
            "top_k": rng.choice([0, 5, 20], T).astype(np.int32),
            "top_p": rng.choice([1.0, 0.9, 0.5], T).astype(np.float32),
            "min_p": rng.choice([0.0, 0.1], T).astype(np.float32)}
    ref = oracle.forward(None, None, rows, s=s)
    lp, inside = oracle.logprob_on_prefix(s, rows, ref["size"])
    assert np.array_equal(inside, ref["in_support"])
    np.testing.assert_array_equal(lp, ref["logprob"])


def test_prefix_logprob_hand_worked():
    # weights [4, 2, 1, 1] (ids 2 and 3 tie); target id 1
    s = np.log(np.array([[4.0, 2.0, 1.0, 1.0]]))
    rows = {"target": np.array([1]), "temperature": np.ones(1, np.float32)}
    lp, inside = oracle.logprob_on_prefix(s, rows, np.array([3]))
    assert inside[0] and abs(lp[0] - math.log(2.0 / 7.0)) < 1e-12  # support {0, 1, 2}
    lp, inside = oracle.logprob_on_prefix(s, rows, np.array([1]))
    assert not inside[0] and lp[0] == -math.inf  # support {0}
    rows["target"] = np.array([3])
    lp, inside = oracle.logprob_on_prefix(s, rows, np.array([3]))
    assert not inside[0]  # the tie puts id 2 before id 3
