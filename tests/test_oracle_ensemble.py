"""Pins of the ensemble majority vote (oracle/ensemble.py)."""
import numpy as np

from oracle import ensemble as E


def test_worked_example():
    # columns: 3 of 4 say yes; 1 of 4; a 2-2 tie with positive margin; a 2-2 tie
    # with negative margin; every expert exactly at the threshold (no votes)
    s = np.array([[0.5, -1.0, 2.0, 0.1, 0.0],
                  [0.2, -0.5, 1.0, 0.2, 0.0],
                  [-0.1, 0.3, -0.5, -1.0, 0.0],
                  [0.9, -0.2, -1.0, -0.1, 0.0]])
    d, v = E.majority_vote(s)
    assert v.tolist() == [3, 1, 2, 2, 0]
    assert d.tolist() == [1, 0, 1, 0, 0]


def test_single_expert_is_its_own_class():
    rng = np.random.default_rng(0)
    s = rng.normal(size=(1, 50)).astype(np.float32)
    d, v = E.majority_vote(s, 0.25)
    assert np.array_equal(d, (s[0] > np.float32(0.25)).astype(np.int32))
    assert np.array_equal(v, d)


def test_threshold_shift_and_expert_order():
    """Shifting scores and threshold together changes nothing away from
    ties; permuting experts changes nothing at all for odd K."""
    rng = np.random.default_rng(1)
    s = rng.normal(size=(5, 200)).astype(np.float32)
    d, v = E.majority_vote(s, 0.0)
    d2, v2 = E.majority_vote(s + np.float32(3.0), 3.0)
    assert np.array_equal(v, v2) and np.array_equal(d, d2)
    d3, v3 = E.majority_vote(s[[4, 2, 0, 1, 3]], 0.0)
    assert np.array_equal(d, d3) and np.array_equal(v, v3)
    # odd K: the decision is the plain majority
    assert np.array_equal(d, (2 * v > 5).astype(np.int32))
