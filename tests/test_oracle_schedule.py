"""Pins for the oracle's DP batch scheduler: exhaustive search over all set
partitions for small queues, closed forms, and validity of the schedule."""
import math

import numpy as np
import pytest

from oracle import schedule as S


def test_set_partitions_counts_are_bell_numbers():
    bell = [1, 1, 2, 5, 15, 52, 203, 877, 4140, 21147]
    for n, b in enumerate(bell):
        assert sum(1 for _ in S.set_partitions(n)) == b


def _random_table(rng, bmax, lmax):
    # non-decreasing in L, arbitrary in b
    t = rng.integers(0, 50, size=(bmax, lmax)).cumsum(axis=1) + rng.integers(1, 200, size=(bmax, 1))
    return t


@pytest.mark.parametrize("seed", range(6))
def test_dp_cost_equals_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    for n in range(1, 9):
        lengths = rng.integers(1, 12, size=n)
        for bmax in (1, 2, 3, 64):
            for cost in (S.linear_cost(rng.integers(0, 300), rng.integers(1, 10)),
                         S.table_cost(_random_table(rng, max(bmax, n), 12))):
                batch, c = S.schedule_dp(lengths, bmax, cost)
                assert c == S.brute_force_cost(lengths, bmax, cost)
                assert S.schedule_cost(lengths, batch, cost) == c


@pytest.mark.slow
def test_dp_cost_equals_exhaustive_search_n10_with_ties():
    rng = np.random.default_rng(99)
    for lengths in (np.array([5, 5, 5, 2, 2, 9, 9, 1, 5, 2]), rng.integers(1, 6, size=10)):
        for bmax, cost in ((3, S.linear_cost(40, 3)), (10, S.linear_cost(100, 1)),
                           (4, S.table_cost(_random_table(rng, 10, 10)))):
            _, c = S.schedule_dp(lengths, bmax, cost)
            assert c == S.brute_force_cost(lengths, bmax, cost)


def _check_valid(lengths, batch, bmax):
    nb = int(batch.max()) + 1 if len(batch) else 0
    assert set(np.unique(batch)) == set(range(nb))
    maxes = [lengths[batch == b].max() for b in range(nb)]
    assert all(np.diff(maxes) >= 0)                        # execution order: ascending max length
    assert all((batch == b).sum() <= bmax for b in range(nb))
    # contiguous in (length, index) order
    order = S.sorted_order(lengths)
    assert all(np.diff(batch[order]) >= 0)


def test_schedule_is_valid_on_a_large_stream():
    rng = np.random.default_rng(5)
    lengths = rng.integers(2, 101, size=3000)
    batch, c = S.schedule_dp(lengths, 64, S.linear_cost(20000, 1))
    _check_valid(lengths, batch, 64)
    assert S.schedule_cost(lengths, batch, S.linear_cost(20000, 1)) == c


def test_pure_overhead_cost_packs_minimum_number_of_batches():
    rng = np.random.default_rng(6)
    for n, bmax in ((1, 4), (10, 3), (130, 64), (64, 64)):
        lengths = rng.integers(1, 100, size=n)
        batch, c = S.schedule_dp(lengths, bmax, S.linear_cost(7, 0))
        assert int(batch.max()) + 1 == math.ceil(n / bmax)
        assert c == 7 * math.ceil(n / bmax)


def test_no_overhead_cost_gives_singletons_or_equal_length_groups():
    # with c0 = 0 a batch of equal lengths costs the same as its singletons.
    # Sorted lengths 1,3,3,3,7 with bmax 2: dp = 1, 4, 7, 10, 17 with choices
    # j = 0, 1, 1 (tie 1 vs 2), 2 (tie 2 vs 3), 4; walking back from 5 gives
    # segments {1}, {3}, {3, 3}, {7}.
    lengths = np.array([3, 3, 3, 7, 1])
    batch, c = S.schedule_dp(lengths, 2, S.linear_cost(0, 1))
    assert c == 3 + 3 + 3 + 7 + 1
    order = [int(batch[i]) for i in S.sorted_order(lengths)]
    assert order == [0, 1, 2, 2, 3]


def test_stable_sort_breaks_length_ties_by_index():
    assert S.sorted_order(np.array([4, 2, 4, 2])).tolist() == [1, 3, 0, 2]


def test_empty_queue():
    batch, c = S.schedule_dp(np.array([], dtype=np.int32), 4, S.linear_cost(1, 1))
    assert batch.size == 0 and c == 0


# --- latency-aware variants -------------------------------------------------------

def test_compositions_count():
    assert [len(list(S.compositions(n))) for n in range(1, 8)] == [2 ** (n - 1) for n in range(1, 8)]


def test_latency_and_cap_worked_example():
    """Four requests of length 5, T(b, L) = 2 + b*L, Bmax 4.  By hand:
    throughput puts all four in one batch (cost 22); summed completion times
    of the eight batchings of the sorted queue are [4] 88, [3,1] 75, [1,3] 79,
    [2,2] 72, [2,1,1] 69, [1,2,1] 71, [1,1,2] 73, [1,1,1,1] 70, so the latency
    objective takes [2,1,1]; a cap of 15 forbids 22 and 17, so throughput
    takes [2,2] (24)."""
    lens = np.array([5, 5, 5, 5])
    cost = S.linear_cost(2, 1)
    b, c = S.schedule_dp(lens, 4, cost)
    assert b.tolist() == [0, 0, 0, 0] and c == 22
    b, c = S.schedule_dp(lens, 4, cost, objective=S.LATENCY)
    assert b.tolist() == [0, 0, 1, 2] and c == 69
    assert S.latency_cost(lens, b, cost) == 69
    b, c = S.schedule_dp(lens, 4, cost, max_cost=15)
    assert b.tolist() == [0, 0, 1, 1] and c == 24


@pytest.mark.parametrize("seed", range(12))
def test_latency_dp_equals_enumeration_of_sorted_batchings(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 11))
    lens = rng.integers(1, 30, n)
    bmax = int(rng.integers(1, n + 1))
    cost = S.linear_cost(int(rng.integers(0, 60)), int(rng.integers(0, 4)))
    cap = int(rng.integers(0, 120)) if seed % 2 else 0
    b, c = S.schedule_dp(lens, bmax, cost, objective=S.LATENCY, max_cost=cap)
    assert c == S.brute_force_sorted(lens, bmax, cost, S.LATENCY, cap)
    assert c == S.latency_cost(lens, b, cost)
    # the batches are consecutive runs of the sorted queue, numbered in order
    order = S.sorted_order(lens)
    assert np.all(np.diff(b[order]) >= 0) and np.all(np.diff(b[order]) <= 1)


@pytest.mark.parametrize("seed", range(8))
def test_capped_throughput_dp_equals_exhaustive_search(seed):
    rng = np.random.default_rng(200 + seed)
    n = int(rng.integers(1, 9))
    lens = rng.integers(1, 12, n)
    bmax = int(rng.integers(1, n + 1))
    cost = S.linear_cost(int(rng.integers(0, 30)), int(rng.integers(1, 4)))
    cap = int(rng.integers(1, 80))
    b, c = S.schedule_dp(lens, bmax, cost, max_cost=cap)
    assert c == S.brute_force_cost(lens, bmax, cost, max_cost=cap)
    assert c == S.schedule_cost(lens, b, cost)
    for k in np.unique(b):
        members = lens[b == k]
        assert len(members) == 1 or cost(len(members), int(members.max())) <= cap
