"""Pins for the oracle's Softmax, LayerNorm and GELU.

Each check uses something other than the oracle itself: invariants that the
mathematics fixes, closed forms, and independent library routines (scipy,
torch) in float64.
"""
import numpy as np
import pytest
import scipy.special
import torch

from oracle import scorer as O


def _rng(seed=0):
    return np.random.default_rng(seed)


# --- softmax -----------------------------------------------------------------

def test_softmax_rows_sum_to_one_and_masked_are_zero():
    r = _rng(1)
    s = r.normal(0, 3, size=(50, 37))
    allowed = r.random((50, 37)) < 0.6
    allowed[:, 5] = True
    p = O.softmax_masked(s, allowed)
    assert np.all(p[~allowed] == 0.0)
    assert np.max(np.abs(p.sum(-1) - 1.0)) <= 1e-14
    assert np.all(p[allowed] > 0)


def test_softmax_shift_invariance():
    r = _rng(2)
    s = r.normal(0, 2, size=(20, 64))
    allowed = np.tril(np.ones((20, 64), dtype=bool), k=10)
    p0 = O.softmax_masked(s, allowed)
    p1 = O.softmax_masked(s + r.normal(0, 50, size=(20, 1)), allowed)
    assert np.max(np.abs(p0 - p1)) <= 1e-13


def test_softmax_matches_scipy_on_allowed_entries():
    r = _rng(3)
    s = r.normal(0, 4, size=(30, 25))
    lens = r.integers(1, 26, size=30)
    allowed = np.arange(25)[None, :] < lens[:, None]
    p = O.softmax_masked(s, allowed)
    for i in range(30):
        ref = scipy.special.softmax(s[i, :lens[i]])
        assert np.max(np.abs(p[i, :lens[i]] - ref)) <= 1e-15
        assert np.all(p[i, lens[i]:] == 0)


def test_softmax_single_allowed_entry_is_one():
    s = np.array([[3.0, -1e300, 7.0]])
    p = O.softmax_masked(s, np.array([[False, True, False]]))
    assert p.tolist() == [[0.0, 1.0, 0.0]]


def test_softmax_large_scores_do_not_overflow():
    s = np.array([[1000.0, 999.0, 998.0]])
    p = O.softmax_masked(s, np.ones_like(s, dtype=bool))
    e = np.exp([0.0, -1.0, -2.0])
    assert np.max(np.abs(p[0] - e / e.sum())) <= 1e-15


# --- LayerNorm ---------------------------------------------------------------

def test_layernorm_pre_affine_moments():
    r = _rng(4)
    y = r.normal(3.0, 2.5, size=(40, 312))
    eps = 1e-12
    z = O.layer_norm(y, np.ones(312), np.zeros(312), eps)
    assert np.max(np.abs(z.mean(-1))) <= 1e-14
    var = y.var(-1)
    assert np.max(np.abs(z.var(-1) - var / (var + eps))) <= 1e-13


def test_layernorm_constant_row_gives_bias():
    y = np.full((3, 64), 7.25)
    g = _rng(5).normal(size=64)
    b = _rng(6).normal(size=64)
    z = O.layer_norm(y, g, b, 1e-5)
    assert np.max(np.abs(z - b)) == 0.0


def test_layernorm_matches_torch():
    r = _rng(7)
    y = r.normal(0, 1.7, size=(33, 768))
    g = 1 + r.normal(0, 0.1, size=768)
    b = r.normal(0, 0.1, size=768)
    for eps in (1e-12, 1e-5):
        z = O.layer_norm(y, g, b, eps)
        ref = torch.nn.functional.layer_norm(torch.from_numpy(y), (768,), torch.from_numpy(g),
                                             torch.from_numpy(b), eps).numpy()
        assert np.max(np.abs(z - ref)) <= 1e-12


def test_layernorm_uses_biased_variance():
    # two values a, -a: biased variance a^2, so (a - 0)/sqrt(a^2) = 1 exactly (eps=0)
    y = np.array([[2.0, -2.0]])
    z = O.layer_norm(y, np.ones(2), np.zeros(2), 0.0)
    assert z.tolist() == [[1.0, -1.0]]


# --- GELU --------------------------------------------------------------------

def test_gelu_closed_forms():
    assert O.gelu(np.array([0.0]))[0] == 0.0
    x = np.linspace(-6, 6, 241)
    # Phi(-x) = 1 - Phi(x)  =>  GELU(-x) = GELU(x) - x
    assert np.max(np.abs(O.gelu(-x) - (O.gelu(x) - x))) <= 1e-14
    # GELU(1) = Phi(1) = 0.8413447460685429...
    assert abs(O.gelu(np.array([1.0]))[0] - 0.8413447460685429) <= 1e-15
    assert abs(O.gelu(np.array([30.0]))[0] - 30.0) <= 1e-12


def test_gelu_matches_torch_both_forms():
    x = np.linspace(-8, 8, 1001)
    t = torch.from_numpy(x)
    assert np.max(np.abs(O.gelu(x, O.GELU_ERF) - torch.nn.functional.gelu(t).numpy())) <= 1e-14
    assert np.max(np.abs(O.gelu(x, O.GELU_TANH)
                         - torch.nn.functional.gelu(t, approximate="tanh").numpy())) <= 1e-14


def test_gelu_erf_against_scipy_normal_cdf():
    x = np.linspace(-5, 5, 101)
    assert np.max(np.abs(O.gelu(x) - x * scipy.special.ndtr(x))) <= 1e-15
