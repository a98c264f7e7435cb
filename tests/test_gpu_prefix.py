"""Shared-prefix best-of-N / pairwise scoring (rm_score_prefix) against the
oracle, which scores every prefix + candidate as its own sequence, and
against rm_score on the same concatenations."""
import numpy as np
import pytest
import torch

import synth
import classifier_scoring_b200 as rm
from oracle import best_of_n as B
from tests.helpers import SCORE_ATOL, config_for, oracle_model

pytestmark = pytest.mark.gpu

DEC = synth.ModelShape(synth.DEC_PRELN, 3, 256, 4, 1024, 5000, 600, synth.W_BF16, synth.GELU_ERF, 1e-5)


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


@pytest.fixture(scope="module")
def flat():
    return synth.make_weights(DEC, 9)


@pytest.fixture(scope="module")
def scorer(flat):
    cfg = config_for(DEC, max_batch_seqs=32, max_tokens=4096, max_len=600)
    with rm.Scorer(cfg, flat) as sc:
        yield sc


def layout(prefix_len, n_cand, seed):
    rng = np.random.default_rng(seed)
    cand_len = rng.integers(1, 90, int(np.sum(n_cand)))
    T = int(np.sum(prefix_len) + cand_len.sum())
    ids = synth.make_token_ids(T, DEC.vocab, seed + 1)
    return ids, cand_len


def run_prefix(sc, ids, prefix_len, n_cand, cand_len):
    nc, ng = int(np.sum(n_cand)), len(n_cand)
    ids_d = torch.from_numpy(ids.astype(np.int32)).cuda()
    out = torch.full((nc,), float("nan"), device="cuda")
    best = torch.full((ng,), -7, dtype=torch.int32, device="cuda")
    lo = torch.full((ng,), float("nan"), device="cuda")
    sc.score_prefix(ids_d, prefix_len, n_cand, cand_len, out, best, lo)
    torch.cuda.synchronize()
    return (out.cpu().numpy().astype(np.float64), best.cpu().numpy(),
            lo.cpu().numpy().astype(np.float64))


def concatenations(ids, prefix_len, n_cand, cand_len):
    seqs = [np.concatenate([p, c]) for p, cs in B.split_groups(ids, prefix_len, n_cand, cand_len)
            for c in cs]
    return np.concatenate(seqs).astype(np.int32), synth.offsets_from_lengths([len(s) for s in seqs])


# prefixes across 64-row blocks, a group without prefix, single-candidate groups,
# candidates longer than one 64-row block
CASES = {
    "mixed": ([37, 0, 64, 130, 1], [3, 1, 2, 4, 2]),
    "pairs": ([200, 90, 5], [2, 2, 2]),
    "long-prefix": ([500], [5]),
}


@pytest.mark.parametrize("case", list(CASES))
def test_prefix_scores_match_oracle_and_unshared_path(scorer, flat, case):
    prefix_len, n_cand = CASES[case]
    ids, cand_len = layout(prefix_len, n_cand, 31 + len(case))
    if case == "long-prefix":
        cand_len = np.minimum(cand_len, 100)
        ids = ids[:int(np.sum(prefix_len) + cand_len.sum())]
    got, best, lo = run_prefix(scorer, ids, prefix_len, n_cand, cand_len)
    ref = B.score_candidates(oracle_model(DEC, flat), ids, prefix_len, n_cand, cand_len)
    assert np.max(np.abs(got - ref)) <= SCORE_ATOL
    # the same concatenations through rm_score, the prefix recomputed per
    # candidate: the same projections, but another attention kernel (packed-row
    # tiles rather than the per-segment prefix kernel), whose online softmax
    # rounds P to bf16 against running maxima over other key blocks; half the
    # score tolerance bounds the difference
    cat_ids, cat_off = concatenations(ids, prefix_len, n_cand, cand_len)
    plain = torch.full((len(cat_off) - 1,), float("nan"), device="cuda")
    scorer.score(torch.from_numpy(cat_ids).cuda(), cat_off, plain)
    torch.cuda.synchronize()
    assert np.max(np.abs(got - plain.cpu().numpy())) <= SCORE_ATOL / 2
    # selection on the kernel's own fp32 scores: the oracle's rule, same decision
    b_ref, lo_ref = B.select(got, n_cand)
    assert best.tolist() == b_ref.tolist()
    assert np.allclose(lo, lo_ref, rtol=1e-6, atol=1e-6)


def test_best_and_logodds_are_optional(scorer):
    prefix_len, n_cand = [10, 20], [2, 3]
    ids, cand_len = layout(prefix_len, n_cand, 41)
    ids_d = torch.from_numpy(ids.astype(np.int32)).cuda()
    out = torch.empty(5, device="cuda")
    scorer.score_prefix(ids_d, prefix_len, n_cand, cand_len, out)
    torch.cuda.synchronize()
    full, _, _ = run_prefix(scorer, ids, prefix_len, n_cand, cand_len)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), full)


def test_invalid_prefix_calls(scorer, flat):
    ids_d = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = torch.empty(4, device="cuda")
    with pytest.raises(rm.RmError):                       # an empty candidate
        scorer.score_prefix(ids_d, [3], [2], [0, 2], out)
    with pytest.raises(rm.RmError):                       # a group without candidates
        scorer.score_prefix(ids_d, [3], [0], [], out)
    with pytest.raises(rm.RmError):                       # prefix + candidate beyond max_len
        scorer.score_prefix(ids_d, [590], [1], [20], out)
    enc = synth.TINY
    with rm.Scorer(config_for(enc), synth.make_weights(enc, 0)) as e:
        with pytest.raises(rm.RmError):                   # the encoder's prefix sees the candidate
            e.score_prefix(ids_d, [3], [1], [2], out)


@pytest.mark.slow
def test_gpt_1p3b_best_of_8_every_candidate_against_the_stored_oracle():
    """The best-of-8 workload at the 1.3B shape (8 posts of 208..512 tokens, 8
    summaries of 24..48 each): every candidate's score, shared prefix and
    unshared concatenation alike, within the score tolerance of the fp64
    oracle's stored scores (tests/golden/make_golden.py; one candidate is
    re-scored here to tie the file to the oracle); each group's choice is the
    first maximum of the kernel's own scores."""
    import os
    from oracle import scorer as O
    w = synth.PREFIX_WORKLOADS["gpt-1.3b-best-of-8"]
    s = w.shape
    ids, prefix_len, n_cand, cand_len = synth.make_prefix_groups(w)
    gold = np.loadtxt(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                   "gpt_1p3b_best_of_8_scores.txt"))
    nc, ng = int(n_cand.sum()), len(n_cand)
    assert gold.shape == (nc,)
    cat_ids, cat_off = concatenations(ids, prefix_len, n_cand, cand_len)
    big = synth.make_weights(s, w.weight_seed)
    cfg = config_for(s, max_batch_seqs=ng + nc, max_tokens=int(cat_off[-1]),
                     max_len=int(np.diff(cat_off).max()))
    with rm.Scorer(cfg, big) as sc:
        got, best, lo = run_prefix(sc, ids, prefix_len, n_cand, cand_len)
        plain = torch.full((nc,), float("nan"), device="cuda")
        sc.score(torch.from_numpy(cat_ids).cuda(), cat_off, plain)
        torch.cuda.synchronize()
        plain = plain.cpu().numpy().astype(np.float64)
    e_shared, e_plain = np.abs(got - gold), np.abs(plain - gold)
    print(f"\ngpt-1.3b-best-of-8: max |gpu - oracle| shared {e_shared.max():.3e}, "
          f"unshared {e_plain.max():.3e} over {nc} candidates")
    assert e_shared.max() <= SCORE_ATOL and e_plain.max() <= SCORE_ATOL
    b_ref, lo_ref = B.select(got, n_cand)
    assert best.tolist() == b_ref.tolist()
    assert np.allclose(lo, lo_ref, rtol=1e-6, atol=1e-6)
    m = oracle_model(s, big)
    del big
    k = int(np.argmin(np.diff(cat_off)))
    assert abs(O.score_one(m, cat_ids[cat_off[k]:cat_off[k + 1]]) - gold[k]) <= 1e-9
