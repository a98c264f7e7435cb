"""Writes the stored expected values under tests/golden/ from the fp64 oracle.

    python tests/golden/make_golden.py

Only the seeded generators (synth) and the oracle are used.  Files:
  tiny_enc_scores.txt -- scores of the 4-sequence tiny encoder workload
                         (2 layers, hidden 128, 2 heads, FFN 512, fp32
                         weights N(0, 0.02), lengths U[8, 32], seed 0).
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import synth  # noqa: E402
from oracle import scorer  # noqa: E402


def tiny_enc_scores():
    w = synth.WORKLOADS["tiny-enc"]
    s = w.shape
    flat = synth.make_weights(s, w.seed)
    m = scorer.unpack_weights(flat, s.arch, s.n_layers, s.hidden, s.n_heads, s.ffn, s.vocab,
                              s.max_pos, s.weight_dtype, s.gelu, s.ln_eps)
    st = synth.make_stream(w)
    ids, off = synth.pack(st, np.arange(len(st.lengths)))
    return scorer.score_packed(m, ids, off)


if __name__ == "__main__":
    np.savetxt(os.path.join(HERE, "tiny_enc_scores.txt"), tiny_enc_scores(), fmt="%.17g",
               header="fp64 oracle scores, tiny-enc workload (seed 0), one per sequence")
    print("written")
