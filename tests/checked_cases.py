"""Cases run in a child process against the checked build of the library
(librmscore_checked.so, RMSCORE_LIB): see tests/test_gpu_checked.py."""
import json
import os
import sys

import numpy as np
import torch

import synth
import classifier_scoring_b200 as rm
from oracle import best_of_n as B
from oracle import scorer as O
from tests.helpers import config_for, oracle_model


def gpu_scores(sc, ids, off):
    out = torch.full((len(off) - 1,), float("nan"), device="cuda")
    sc.score(torch.from_numpy(ids).cuda(), off, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def valid_inputs():
    """Every kernel of the scorer on consistent inputs: no failed bounds test,
    and the scores of the product build."""
    res = {"checked": rm.build_checked(), "bounds_before": rm.bounds_errors()}
    w = synth.WORKLOADS["tiny-enc"]
    st = synth.make_stream(w)
    ids, off = synth.pack(st, np.arange(len(st.lengths)))
    gold = np.loadtxt(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                   "tiny_enc_scores.txt"))
    for attn in (rm.ATTN_FUSED, rm.ATTN_MATERIALIZED):
        cfg = config_for(w.shape, max_batch_seqs=8, max_tokens=256, max_len=64, attn_impl=attn)
        with rm.Scorer(cfg, synth.make_weights(w.shape, w.seed)) as sc:
            res[f"tiny_err_{attn}"] = float(np.max(np.abs(gpu_scores(sc, ids, off) - gold)))
    # an encoder with rows past 128 tokens: the long-row tensor-core attention
    enc = synth.ModelShape(synth.ENC_POSTLN, 2, 256, 4, 1024, 5000, 600, synth.W_BF16,
                           synth.GELU_ERF, 1e-12)
    eflat = synth.make_weights(enc, 11)
    em = oracle_model(enc, eflat)
    cfg = config_for(enc, max_batch_seqs=16, max_tokens=2048, max_len=600, attn_impl=rm.ATTN_FUSED)
    with rm.Scorer(cfg, eflat) as sc:
        lens = np.array([1, 200, 130, 7, 300])
        o = synth.offsets_from_lengths(lens)
        tids = synth.make_token_ids(int(o[-1]), enc.vocab, 6)
        got = gpu_scores(sc, tids, o)
        want = np.array([O.score_one(em, tids[o[i]:o[i + 1]]) for i in range(len(lens))])
        res["enc_long_err_0"] = float(np.max(np.abs(got - want)))
    # the decoder paths: tiles, materialised, and shared prefixes with the vote of best-of-N
    dec = synth.ModelShape(synth.DEC_PRELN, 2, 256, 4, 1024, 5000, 600, synth.W_BF16,
                           synth.GELU_ERF, 1e-5)
    flat = synth.make_weights(dec, 9)
    m = oracle_model(dec, flat)
    prefix_len, n_cand = np.array([37, 0, 70]), np.array([2, 1, 3])
    rng = np.random.default_rng(3)
    cand_len = rng.integers(1, 40, int(n_cand.sum()))
    pids = synth.make_token_ids(int(prefix_len.sum() + cand_len.sum()), dec.vocab, 4)
    ref = B.score_candidates(m, pids, prefix_len, n_cand, cand_len)
    for attn in (rm.ATTN_FUSED, rm.ATTN_MATERIALIZED):
        cfg = config_for(dec, max_batch_seqs=16, max_tokens=2048, max_len=600, attn_impl=attn)
        with rm.Scorer(cfg, flat) as sc:
            lens = np.array([1, 65, 130, 7])
            o = synth.offsets_from_lengths(lens)
            tids = synth.make_token_ids(int(o[-1]), dec.vocab, 5)
            got = gpu_scores(sc, tids, o)
            want = np.array([O.score_one(m, tids[o[i]:o[i + 1]]) for i in range(len(lens))])
            res[f"dec_err_{attn}"] = float(np.max(np.abs(got - want)))
            out = torch.full((int(n_cand.sum()),), float("nan"), device="cuda")
            best = torch.zeros(len(n_cand), dtype=torch.int32, device="cuda")
            sc.score_prefix(torch.from_numpy(pids).cuda(), prefix_len, n_cand, cand_len, out, best)
            torch.cuda.synchronize()
            res[f"prefix_err_{attn}"] = float(np.max(np.abs(out.cpu().numpy() - ref)))
    res["bounds_after"] = rm.bounds_errors()
    return res


def invalid_metadata():
    """Metadata the kernels' own tests catch in the checked build: a sequence of
    length 0 given to the head (its last-token row would be -1), and a softmax
    told of more tokens than its offsets hold.  Each is counted, the access
    skipped, and the context stays usable."""
    if not rm.build_checked():
        # these inputs are only safe where the kernels test them
        raise SystemExit("invalid_metadata needs the checked build of the library")
    res = {"bounds_before": rm.bounds_errors()}
    H = 128
    x = torch.randn(8, H, device="cuda").to(torch.bfloat16)
    w = torch.randn(H, device="cuda")
    off = torch.tensor([0, 3, 3, 8], dtype=torch.int32, device="cuda")     # sequence 1 is empty
    out = torch.full((3,), float("nan"), device="cuda")
    rm.ops.head(x, off, 3, w, 0.0, H, 1, out)
    torch.cuda.synchronize()
    res["head_bounds"] = rm.bounds_errors()
    res["head_out"] = [float(v) for v in out.cpu().numpy()]
    lens = np.array([5, 9])
    o = synth.offsets_from_lengths(lens)
    rb, so = rm.ops.varlen_meta(o, 2)
    S = torch.randn(int(so[-1]), device="cuda").to(torch.bfloat16)
    rm.ops.softmax(S, rm.BF16, torch.from_numpy(o).cuda(), torch.from_numpy(so).cuda(), 2,
                   int(o[-1]) + 4, 2, 9, 0)                                # 4 tokens too many
    torch.cuda.synchronize()
    res["softmax_bounds"] = rm.bounds_errors()
    # the same context then scores correctly
    res.update({k: v for k, v in valid_inputs().items() if k.startswith("tiny_err")})
    return res


if __name__ == "__main__":
    torch.cuda.set_device(0)
    case = sys.argv[1]
    print(json.dumps(valid_inputs() if case == "valid" else invalid_metadata()))
