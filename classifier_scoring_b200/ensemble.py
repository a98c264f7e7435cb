"""Replica ensemble with majority vote (the SambaNova blog's accuracy section:
several TinyBERT "experts" classify the same input and vote).

Each expert is a scorer handle with its own weights.  On one GPU the experts
score the batch on their own streams at the same time, and rm_op_vote reduces
their [K][n] scores to a decision per input.  Across ranks (one expert per
GPU) the per-rank scores are gathered with torch.distributed before the vote:
4 bytes per input and expert cross the interconnect.  Marshalling only: the
scoring and the vote run in the library's kernels.
"""
from typing import List, Optional, Sequence

from . import ops


class Ensemble:
    """K scorer handles (experts) voting on one GPU."""

    def __init__(self, experts: Sequence, streams: Optional[List] = None):
        import torch
        self.experts = list(experts)
        self.streams = streams or [torch.cuda.Stream() for _ in self.experts]
        self._fork = torch.cuda.Event()
        self._join = [torch.cuda.Event() for _ in self.experts]

    def score_and_vote(self, ids_dev, offsets, scores, decision, votes=None, threshold=0.0,
                       stream=None, plans=None):
        """Every expert scores the packed batch (device ids, host offsets) into
        its row of scores[K][n]; then the vote writes decision[n] (and votes[n])
        on `stream` (default: the current stream), after all experts.  With
        plans (one per expert, from plan()) the experts only enqueue kernels,
        so the whole call can be captured into a CUDA graph."""
        import torch
        main = stream or torch.cuda.current_stream()
        K, n = len(self.experts), len(offsets) - 1
        self._fork.record(main)
        for k, (sc, st) in enumerate(zip(self.experts, self.streams)):
            st.wait_event(self._fork)
            if plans is not None:
                plans[k].score(ids_dev, scores[k], st)
            else:
                sc.score(ids_dev, offsets, scores[k], st)
            self._join[k].record(st)
        for ev in self._join:
            main.wait_event(ev)
        ops.vote(scores, K, n, threshold, decision, votes, main)

    def plan(self, offsets):
        """One rm_plan per expert for this batch shape."""
        return [sc.plan(offsets) for sc in self.experts]


def gather_scores(local_scores, group=None):
    """All ranks' scores of the same n inputs, stacked in rank order: rank k's
    expert in row k of a [world][n] tensor on local_scores' device."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(local_scores) for _ in range(world)]
    dist.all_gather(parts, local_scores, group=group)
    return torch.stack(parts)
