"""Pins of the best-of-N / pairwise oracle (oracle/best_of_n.py) against
hand-worked values and properties of the causal reward model."""
import numpy as np
import pytest

import synth
from oracle import best_of_n as B
from oracle import scorer as O
from tests.helpers import oracle_model

SMALL_DEC = synth.ModelShape(synth.DEC_PRELN, 2, 64, 4, 128, 300, 96, synth.W_F32, synth.GELU_ERF, 1e-5)


def test_select_worked_example():
    # group 0: a tie between candidates 1 and 2 goes to the first; r1 - r0 = 0.2
    # group 1: a single candidate; group 2: the first candidate wins, r1 - r0 < 0
    scores = np.array([0.1, 0.3, 0.3, -1.0, 2.0, 5.0, 4.0])
    best, lo = B.select(scores, [4, 1, 2])
    assert best.tolist() == [1, 0, 0]
    assert np.allclose(lo, [0.2, 0.0, -1.0], atol=1e-15)


def test_split_groups_layout():
    ids = np.arange(16)
    groups = B.split_groups(ids, [3, 0, 2], [2, 1, 3], [1, 2, 4, 1, 1, 2])
    assert [g[0].tolist() for g in groups] == [[0, 1, 2], [], [10, 11]]
    assert [[c.tolist() for c in g[1]] for g in groups] == [[[3], [4, 5]], [[6, 7, 8, 9]],
                                                             [[12], [13], [14, 15]]]
    with pytest.raises(ValueError):
        B.split_groups(np.arange(15), [3, 0, 2], [2, 1, 3], [1, 2, 4, 1, 1, 2])


@pytest.fixture(scope="module")
def model():
    return oracle_model(SMALL_DEC, synth.make_weights(SMALL_DEC, 21))


def test_no_prefix_is_plain_packed_scoring(model):
    lens = np.array([5, 1, 9, 3])
    ids = synth.make_token_ids(int(lens.sum()), SMALL_DEC.vocab, 22)
    got = B.score_candidates(model, ids, [0, 0], [3, 1], lens)
    assert np.array_equal(got, O.score_packed(model, ids, synth.offsets_from_lengths(lens)))


def test_candidates_are_scored_independently(model):
    """Changing one candidate changes only its own score, and reordering a
    group's candidates reorders its scores and its best index."""
    rng = np.random.default_rng(23)
    pre = rng.integers(0, SMALL_DEC.vocab, 11)
    cands = [rng.integers(0, SMALL_DEC.vocab, n) for n in (4, 7, 2)]
    def run(cs):
        ids = np.concatenate([pre] + cs)
        return B.score_candidates(model, ids, [len(pre)], [len(cs)], [len(c) for c in cs])
    base = run(cands)
    changed = run([cands[0], rng.integers(0, SMALL_DEC.vocab, 7), cands[2]])
    assert changed[0] == base[0] and changed[2] == base[2] and changed[1] != base[1]
    perm = [2, 0, 1]
    swapped = run([cands[k] for k in perm])
    assert np.array_equal(swapped, base[perm])
    b0, _ = B.select(base, [3])
    b1, _ = B.select(swapped, [3])
    assert perm[int(b1[0])] == int(b0[0])


def test_prefix_states_do_not_depend_on_the_candidate(model):
    """The identity that makes sharing exact: the causal decoder's hidden
    states of the prefix tokens are the same whatever candidate follows."""
    rng = np.random.default_rng(24)
    pre = rng.integers(0, SMALL_DEC.vocab, 13)
    h_alone = O.hidden_states(model, pre)
    for n in (1, 6):
        c = rng.integers(0, SMALL_DEC.vocab, n)
        h = O.hidden_states(model, np.concatenate([pre, c]))
        assert np.allclose(h[:13], h_alone, rtol=0, atol=1e-12)
