"""rm_plan: launch-only scoring of a prepared batch shape, equal to rm_score,
and replayable from a CUDA graph with new ids; an ensemble captured whole."""
import numpy as np
import pytest
import torch

import synth
import classifier_scoring_b200 as rm
from classifier_scoring_b200.ensemble import Ensemble
from oracle import ensemble as E
from tests.helpers import config_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def batch(shape, lens, seed):
    off = synth.offsets_from_lengths(np.array(lens))
    ids = synth.make_token_ids(int(off[-1]), shape.vocab, seed)
    return torch.from_numpy(ids).cuda(), off


@pytest.mark.parametrize("name", ["tiny-enc", "tinybert-b1"])
def test_plan_equals_rm_score_and_replays_from_a_graph(name):
    w = synth.WORKLOADS[name]
    lens = [5, 31, 17] if name == "tiny-enc" else [128]
    with rm.Scorer(config_for(w.shape, max_len=min(512, w.shape.max_pos)),
                   synth.make_weights(w.shape, w.seed)) as sc:
        ids, off = batch(w.shape, lens, 3)
        n = len(lens)
        ref = torch.full((n,), float("nan"), device="cuda")
        sc.score(ids, off, ref)
        plan = sc.plan(off)
        got = torch.full((n,), float("nan"), device="cuda")
        s = torch.cuda.Stream()
        plan.score(ids, got, s)                       # warm-up outside capture
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        # capture once, replay on new ids written into the same buffer
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            plan.score(ids, got, s)
        for seed in (4, 5):
            new_ids, _ = batch(w.shape, lens, seed)
            ids.copy_(new_ids)
            got.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            sc.score(ids, off, ref)
            torch.cuda.synchronize()
            assert torch.equal(got, ref)
        del g
        plan.close()


def test_ensemble_captured_whole_votes_like_eager():
    shape = synth.TINY
    experts = [rm.Scorer(config_for(shape), synth.make_weights(shape, 7 + 100 * k)) for k in range(4)]
    try:
        ens = Ensemble(experts)
        ids, off = batch(shape, [9, 20, 32, 8, 15], 11)
        K, n = 4, 5
        plans = ens.plan(off)
        s = torch.cuda.Stream()
        scores = torch.zeros(K, n, device="cuda")
        dec = torch.zeros(n, dtype=torch.int32, device="cuda")
        votes = torch.zeros(n, dtype=torch.int32, device="cuda")
        ens.score_and_vote(ids, off, scores, dec, votes, stream=s, plans=plans)   # warm-up
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            ens.score_and_vote(ids, off, scores, dec, votes, stream=s, plans=plans)
        scores.fill_(float("nan"))
        dec.fill_(-1)
        g.replay()
        torch.cuda.synchronize()
        eager_scores = torch.zeros(K, n, device="cuda")
        eager_dec = torch.zeros(n, dtype=torch.int32, device="cuda")
        ens.score_and_vote(ids, off, eager_scores, eager_dec)
        torch.cuda.synchronize()
        assert torch.equal(scores, eager_scores) and torch.equal(dec, eager_dec)
        d_ref, v_ref = E.majority_vote(scores.cpu().numpy())
        assert np.array_equal(dec.cpu().numpy(), d_ref) and np.array_equal(votes.cpu().numpy(), v_ref)
        del g
        for p in plans:
            p.close()
    finally:
        for e in experts:
            e.close()


def test_plan_validates_like_rm_score():
    w = synth.WORKLOADS["tiny-enc"]
    with rm.Scorer(config_for(w.shape), synth.make_weights(w.shape, w.seed)) as sc:
        for bad in ([0, 3, 3], [1, 4], [0, 4000]):
            with pytest.raises(rm.RmError):
                sc.plan(np.array(bad, dtype=np.int32))
