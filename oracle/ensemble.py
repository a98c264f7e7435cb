"""Majority vote over an ensemble of scorer replicas (TEST INFRASTRUCTURE ONLY).

SambaNova blog "Breakthrough efficiency in NLP model deployment", section on
improving accuracy with the DataScale system (Figs. 4 and 5): several
TinyBERT instances ("experts"), one per socket, classify the same input and a
majority vote over their answers gives the ensemble's answer.

The scorer here has a scalar head, so an expert's answer for input i is the
binary class [s_k,i > threshold] (the sign of the logit for threshold 0).
Readings where the page is silent: the vote counts the experts that answer 1;
the ensemble answers 1 when more than half do, 0 when fewer than half do, and
on an exact tie (even K) the sign of the summed margins sum_k (s_k,i -
threshold) decides (1 if it is > 0).  That sum is taken in float32 in expert
order k = 0..K-1, the precision and order of the kernel, because it decides
an integer.
"""
import numpy as np


def majority_vote(scores, threshold: float = 0.0):
    """scores: [K][n] (expert k's score of input i).  Returns (decision int32[n],
    votes int32[n])."""
    s = np.asarray(scores, dtype=np.float32)
    K, n = s.shape
    thr = np.float32(threshold)
    votes = np.zeros(n, dtype=np.int32)
    decision = np.zeros(n, dtype=np.int32)
    for i in range(n):
        v = 0
        margin = np.float32(0.0)
        for k in range(K):
            if s[k, i] > thr:
                v += 1
            margin = np.float32(margin + np.float32(s[k, i] - thr))
        votes[i] = v
        if 2 * v > K:
            decision[i] = 1
        elif 2 * v < K:
            decision[i] = 0
        else:
            decision[i] = 1 if margin > 0 else 0
    return decision, votes
