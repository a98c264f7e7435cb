"""rm_schedule (the product's DP scheduler) is bit-exact with the oracle's DP."""
import numpy as np
import pytest

import synth
import classifier_scoring_b200 as rm
from classifier_scoring_b200 import build
from oracle import schedule as S
from tests.helpers import config_for


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def sched_cfg(bmax, c0, c1, max_len, table=None, objective=0, max_cost=0):
    return config_for(synth.BERT_BASE, max_len=max_len, sched_max_batch=bmax, sched_c0=c0,
                      sched_c1=c1, sched_table=table, sched_objective=objective,
                      sched_max_cost=max_cost)


@pytest.mark.parametrize("name", ["bert-base-len2-100", "bert-base-len5-500"])
def test_workload_streams_bit_exact(name):
    w = synth.WORKLOADS[name]
    lengths = synth.make_stream(w).lengths
    for c0, c1 in ((0, 1), (20000, 1), (5000, 3), (1, 0)):
        cfg = sched_cfg(w.max_batch, c0, c1, 512)
        ours = rm.schedule(cfg, lengths)
        ref, _ = S.schedule_dp(lengths, w.max_batch, S.linear_cost(c0, c1))
        assert np.array_equal(ours, ref)


def test_table_cost_bit_exact():
    rng = np.random.default_rng(3)
    bmax, lmax = 16, 40
    table = rng.integers(0, 30, size=(bmax, lmax)).cumsum(axis=1) + rng.integers(50, 500, size=(bmax, 1))
    lengths = rng.integers(1, lmax + 1, size=2000)
    ours = rm.schedule(sched_cfg(bmax, 0, 0, lmax, table), lengths)
    ref, _ = S.schedule_dp(lengths, bmax, S.table_cost(table))
    assert np.array_equal(ours, ref)


def test_small_queues_with_ties_bit_exact_and_optimal():
    rng = np.random.default_rng(4)
    for n in range(1, 9):
        for _ in range(5):
            lengths = rng.integers(1, 5, size=n)
            for bmax in (1, 2, 3, 8):
                cfg = sched_cfg(bmax, int(rng.integers(0, 20)), int(rng.integers(0, 4)), 8)
                ours = rm.schedule(cfg, lengths)
                cost = S.linear_cost(cfg.sched_c0, cfg.sched_c1)
                ref, c = S.schedule_dp(lengths, bmax, cost)
                assert np.array_equal(ours, ref)
                assert S.schedule_cost(lengths, ours, cost) == S.brute_force_cost(lengths, bmax, cost)


def test_empty_queue_and_errors():
    cfg = sched_cfg(4, 1, 1, 100)
    assert rm.schedule(cfg, []).size == 0
    with pytest.raises(rm.RmError):
        rm.schedule(cfg, [3, 0, 2])
    with pytest.raises(rm.RmError):
        rm.schedule(cfg, [3, 101])
    bad = np.tile(np.arange(100, 0, -1, dtype=np.int64), (4, 1))     # decreasing along L
    with pytest.raises(rm.RmError):
        rm.schedule(sched_cfg(4, 0, 0, 100, bad), [3])


@pytest.mark.parametrize("objective", [S.THROUGHPUT, S.LATENCY], ids=["throughput", "latency"])
@pytest.mark.parametrize("cap", [0, 30000, 120000])
def test_latency_objective_and_cap_bit_exact_on_the_stream(objective, cap):
    w = synth.WORKLOADS["bert-base-len2-100"]
    lengths = synth.make_stream(w, 3000).lengths
    ours = rm.schedule(sched_cfg(64, 20000, 1, 512, objective=objective, max_cost=cap), lengths)
    ref, _ = S.schedule_dp(lengths, 64, S.linear_cost(20000, 1), objective=objective, max_cost=cap)
    assert np.array_equal(ours, ref)


def test_latency_objective_small_queues_bit_exact():
    rng = np.random.default_rng(5)
    for n in range(1, 10):
        for _ in range(4):
            lengths = rng.integers(1, 6, size=n)
            bmax = int(rng.integers(1, n + 1))
            c0, c1 = int(rng.integers(0, 20)), int(rng.integers(0, 4))
            cap = int(rng.integers(0, 40))
            cost = S.linear_cost(c0, c1)
            for objective in (S.THROUGHPUT, S.LATENCY):
                ours = rm.schedule(sched_cfg(bmax, c0, c1, 8, objective=objective, max_cost=cap), lengths)
                ref, c = S.schedule_dp(lengths, bmax, cost, objective=objective, max_cost=cap)
                assert np.array_equal(ours, ref)


def test_latency_knobs_are_validated():
    with pytest.raises(rm.RmError):
        rm.schedule(sched_cfg(4, 1, 1, 100, objective=2), [3])
    with pytest.raises(rm.RmError):
        rm.schedule(sched_cfg(4, 1, 1, 100, max_cost=-1), [3])


def test_default_stream_schedule_matches_the_oracle_and_batch_count():
    """The schedule bench.py runs: the 10,000-request lengths-2..100 stream,
    T(b, L) = 20000 + b*L, Bmax 64 -- bit-exact with the oracle, 157 batches."""
    w = synth.WORKLOADS["bert-base-len2-100"]
    lengths = synth.make_stream(w).lengths
    ours = rm.schedule(sched_cfg(64, 20000, 1, 512), lengths)
    ref, _ = S.schedule_dp(lengths, 64, S.linear_cost(20000, 1))
    assert np.array_equal(ours, ref)
    assert int(ours.max()) + 1 == 157
    assert np.bincount(ours).max() <= 64
