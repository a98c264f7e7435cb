"""The ensemble vote kernel (rm_op_vote) and an ensemble of scorer replicas
on one GPU against the oracle."""
import numpy as np
import pytest
import torch

import synth
import classifier_scoring_b200 as rm
from classifier_scoring_b200.ensemble import Ensemble
from oracle import ensemble as E
from oracle import scorer as O
from tests.helpers import SCORE_ATOL, config_for, oracle_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


@pytest.mark.parametrize("K", [1, 2, 3, 8])
@pytest.mark.parametrize("thr", [0.0, 0.25])
def test_vote_kernel_matches_oracle_bit_exact(K, thr):
    rng = np.random.default_rng(K * 10 + int(thr * 4))
    n = 3001
    # coarse values: exact ties, scores equal to the threshold, zero margins
    s = (rng.integers(-4, 5, size=(K, n)) * 0.25).astype(np.float32)
    s[:, :50] = np.float32(thr)
    sd = torch.from_numpy(s).cuda()
    dec = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    votes = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    rm.ops.vote(sd, K, n, thr, dec, votes)
    torch.cuda.synchronize()
    d_ref, v_ref = E.majority_vote(s, thr)
    assert np.array_equal(votes.cpu().numpy(), v_ref)
    assert np.array_equal(dec.cpu().numpy(), d_ref)


def test_vote_rejects_bad_arguments():
    x = torch.zeros(4, device="cuda")
    with pytest.raises(rm.RmError):
        rm.ops.vote(x, 0, 4)
    with pytest.raises(rm.RmError):
        rm.ops.vote(None, 1, 4)


def test_three_experts_on_one_gpu_vote_like_the_oracle():
    shape = synth.TINY
    seeds = [0, 100, 200]
    flats = [synth.make_weights(shape, s) for s in seeds]
    lens = synth.make_lengths(24, 8, 32, 5)
    off = synth.offsets_from_lengths(lens)
    ids = synth.make_token_ids(int(off[-1]), shape.vocab, 6)
    K, n = len(seeds), len(lens)
    experts = [rm.Scorer(config_for(shape), f) for f in flats]
    try:
        ens = Ensemble(experts)
        scores = torch.full((K, n), float("nan"), device="cuda")
        dec = torch.full((n,), -1, dtype=torch.int32, device="cuda")
        votes = torch.full((n,), -1, dtype=torch.int32, device="cuda")
        ens.score_and_vote(torch.from_numpy(ids).cuda(), off, scores, dec, votes)
        torch.cuda.synchronize()
        got = scores.cpu().numpy()
    finally:
        for e in experts:
            e.close()
    ref = np.stack([O.score_packed(oracle_model(shape, f), ids, off) for f in flats])
    assert np.max(np.abs(got - ref)) <= SCORE_ATOL
    # the vote on the kernel's own fp32 scores: the oracle's rule, same decisions
    d_ref, v_ref = E.majority_vote(got)
    assert np.array_equal(dec.cpu().numpy(), d_ref) and np.array_equal(votes.cpu().numpy(), v_ref)
    # and on the oracle's scores wherever no expert sits within the tolerance of 0
    clear = np.all(np.abs(ref) > 2 * SCORE_ATOL, axis=0)
    d_o, _ = E.majority_vote(ref)
    assert np.array_equal(dec.cpu().numpy()[clear], d_o[clear])
