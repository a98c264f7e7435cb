"""Writes the stored expected values under tests/golden/ from the fp64 oracle.

    python tests/golden/make_golden.py [name ...]     (default: every file)

Only the seeded generators (synth) and the oracle are used.  Files:
  tiny_enc_scores.txt -- scores of the 4-sequence tiny encoder workload
                         (2 layers, hidden 128, 2 heads, FFN 512, fp32
                         weights N(0, 0.02), lengths U[8, 32], seed 0).
  gpt_1p3b_rm_batch_scores.txt -- scores of every sequence of the first
                         64-sequence batch of the 1.3B-shape causal reward
                         model stream (24 layers, d 2048, 16 heads, FFN 8192,
                         bf16 weights, lengths U[256, 560], seed 4).
  gpt_1p3b_best_of_8_scores.txt -- scores of all 64 candidates of the
                         best-of-8 workload (8 posts of U[208, 512] tokens, 8
                         summaries of U[24, 48] each, the 1.3B-shape weights
                         of seed 4, requests of seed 5), each candidate scored
                         as its own post + summary sequence.
  bert_base_len5_500_longest_batch_scores.txt -- request index and score of
                         every sequence of the last (longest) DP batch of the
                         10,000-request BERT-base stream with lengths
                         U[5, 500] (seed 3), scheduled with Bmax 32 and the
                         cost c0 + c1*b*L, c0 = 20000, c1 = 1.
"""
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import synth  # noqa: E402
from oracle import best_of_n as OB  # noqa: E402
from oracle import schedule as OS  # noqa: E402
from oracle import scorer  # noqa: E402


def _model(name):
    w = synth.WORKLOADS[name]
    s = w.shape
    flat = synth.make_weights(s, w.seed)
    return scorer.unpack_weights(flat, s.arch, s.n_layers, s.hidden, s.n_heads, s.ffn, s.vocab,
                                 s.max_pos, s.weight_dtype, s.gelu, s.ln_eps)


def _score_all(m, ids, off, label):
    out = np.empty(len(off) - 1)
    t0 = time.time()
    for i in range(len(off) - 1):
        out[i] = scorer.score_one(m, ids[off[i]:off[i + 1]])
        print(f"{label}: {i + 1}/{len(out)} ({time.time() - t0:.0f} s)", flush=True)
    return out


def tiny_enc_scores():
    w = synth.WORKLOADS["tiny-enc"]
    st = synth.make_stream(w)
    ids, off = synth.pack(st, np.arange(len(st.lengths)))
    return scorer.score_packed(_model("tiny-enc"), ids, off)


def gpt_1p3b_batch():
    """Packed ids and offsets of the first 64 requests of the gpt-1.3b-rm stream."""
    w = synth.WORKLOADS["gpt-1.3b-rm"]
    st = synth.make_stream(w)
    return synth.pack(st, np.arange(w.max_batch))


def bert_base_len5_500_longest_batch():
    """Request indices of the last DP batch of the full lengths-5-500 stream,
    with its packed ids and offsets."""
    w = synth.WORKLOADS["bert-base-len5-500"]
    st = synth.make_stream(w)
    batch, _ = OS.schedule_dp(st.lengths, w.max_batch, OS.linear_cost(20000, 1))
    idx = np.nonzero(batch == batch.max())[0]
    ids, off = synth.pack(st, idx)
    return idx, ids, off


def gpt_best_of_8_scores():
    w = synth.PREFIX_WORKLOADS["gpt-1.3b-best-of-8"]
    ids, prefix_len, n_cand, cand_len = synth.make_prefix_groups(w)
    m = _model("gpt-1.3b-rm")
    out = []
    for p, cands in OB.split_groups(ids, prefix_len, n_cand, cand_len):
        for c in cands:
            out.append(scorer.score_one(m, np.concatenate([p, c])))
            print(f"best-of-8: {len(out)}/{int(n_cand.sum())}", flush=True)
    return np.array(out)


def write(name):
    path = os.path.join(HERE, name)
    if name == "tiny_enc_scores.txt":
        np.savetxt(path, tiny_enc_scores(), fmt="%.17g",
                   header="fp64 oracle scores, tiny-enc workload (seed 0), one per sequence")
    elif name == "gpt_1p3b_rm_batch_scores.txt":
        ids, off = gpt_1p3b_batch()
        s = _score_all(_model("gpt-1.3b-rm"), ids, off, name)
        np.savetxt(path, s, fmt="%.17g",
                   header="fp64 oracle scores, gpt-1.3b-rm workload (seed 4), first 64 requests, "
                          "one per sequence")
    elif name == "gpt_1p3b_best_of_8_scores.txt":
        np.savetxt(path, gpt_best_of_8_scores(), fmt="%.17g",
                   header="fp64 oracle scores, gpt-1.3b-best-of-8 (weights seed 4, requests seed 5), "
                          "every candidate as its own prefix + candidate sequence, group-major")
    elif name == "bert_base_len5_500_longest_batch_scores.txt":
        idx, ids, off = bert_base_len5_500_longest_batch()
        s = _score_all(_model("bert-base-len5-500"), ids, off, name)
        np.savetxt(path, np.column_stack([idx.astype(np.float64), s]), fmt=["%d", "%.17g"],
                   header="request index, fp64 oracle score; bert-base-len5-500 (seed 3), last DP "
                          "batch (Bmax 32, cost 20000 + b*L)")
    else:
        raise SystemExit(f"unknown golden file {name}")
    print("written", path)


ALL = ["tiny_enc_scores.txt", "gpt_1p3b_rm_batch_scores.txt",
       "bert_base_len5_500_longest_batch_scores.txt", "gpt_1p3b_best_of_8_scores.txt"]

if __name__ == "__main__":
    for n in (sys.argv[1:] or ALL):
        write(n)
