"""Best-of-N and pairwise scoring of candidates that share a prefix
(TEST INFRASTRUCTURE ONLY).

"Learning to summarize from human feedback" (summary page, method-adaptation
section): the reward model is the supervised GPT-style baseline with a scalar
head, trained so that the difference of two summaries' scores is the log-odds
that one is preferred over the other; best-of-N rejection sampling draws N
summaries of one post, scores each with the reward model and keeps the
highest.  A summary's score is the reward model's score of the sequence
post + summary.

This module states that with no sharing at all: every candidate is scored as
its own concatenated sequence by ``scorer.score_one``.  Whatever the fast path
shares between candidates must reproduce these numbers.
"""
import numpy as np

from oracle import scorer


def split_groups(ids, prefix_len, n_cand, cand_len):
    """The packed layout of a shared-prefix call: per group g, prefix_len[g]
    prefix tokens, then its n_cand[g] candidates.  Returns, per group,
    (prefix ids, [candidate ids ...])."""
    ids = np.asarray(ids)
    groups, pos, k = [], 0, 0
    for g in range(len(prefix_len)):
        pre = ids[pos:pos + int(prefix_len[g])]
        pos += int(prefix_len[g])
        cands = []
        for _ in range(int(n_cand[g])):
            cands.append(ids[pos:pos + int(cand_len[k])])
            pos += int(cand_len[k])
            k += 1
        groups.append((pre, cands))
    if pos != len(ids) or k != len(cand_len):
        raise ValueError("layout does not cover the ids exactly")
    return groups


def score_candidates(m, ids, prefix_len, n_cand, cand_len) -> np.ndarray:
    """Score of prefix + candidate for every candidate, in packed order."""
    out = []
    for pre, cands in split_groups(ids, prefix_len, n_cand, cand_len):
        for c in cands:
            out.append(scorer.score_one(m, np.concatenate([pre, c])))
    return np.array(out, dtype=np.float64)


def select(scores, n_cand):
    """Per group: the index of the highest score (the first one on ties) and
    r_1 - r_0, the pairwise log-odds of the group's first two candidates (0
    for a single candidate)."""
    best, logodds, a = [], [], 0
    for n in n_cand:
        r = [float(v) for v in scores[a:a + int(n)]]
        i_best = 0
        for i in range(1, len(r)):
            if r[i] > r[i_best]:
                i_best = i
        best.append(i_best)
        logodds.append(r[1] - r[0] if len(r) >= 2 else 0.0)
        a += int(n)
    return np.array(best, dtype=np.int64), np.array(logodds, dtype=np.float64)
