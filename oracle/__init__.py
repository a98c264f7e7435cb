"""fp64 CPU oracle for the transformer scorer and the DP batch scheduler.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import this package.  The
product (``classifier_scoring_b200``) never imports it, and this package
imports nothing from the product: the two share no code.  The seeded inputs
both sides consume come from ``synth``, which holds none of the method's
arithmetic.

Contents:
  scorer    -- plain fp64 forward pass of the compact encoder (post-LN,
               BERT/TinyBERT-style) and of the GPT-style pre-LN causal reward
               model, per sequence (padding-free) and padded-with-mask.
  schedule  -- the dynamic-programming batch scheduler and an exhaustive
               search over all set partitions for small queues.
  best_of_n -- best-of-N / pairwise scoring of candidates that share a
               prefix, each scored as its own concatenated sequence.
  ensemble  -- majority vote of scorer replicas ("experts") on the binary
               class of their scores.

Every function cites the page passage it follows.  Pins (tests that check
this package against something other than itself) live in
``tests/test_oracle_*.py``.  Parity status: every function here is pinned;
none is "parity unpinned".
"""
