"""End-to-end parity of rm_score against the fp64 oracle on every workload,
plus edge cases, error paths and the host-buffer entry point."""
import functools
import os

import numpy as np
import pytest
import torch

import synth
import classifier_scoring_b200 as rm
from oracle import schedule as OS
from tests.helpers import SCORE_ATOL, config_for, oracle_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


@functools.lru_cache(maxsize=4)
def weights(name):
    w = synth.WORKLOADS[name]
    return synth.make_weights(w.shape, w.seed)


@functools.lru_cache(maxsize=2)
def omodel(name):
    return oracle_model(synth.WORKLOADS[name].shape, weights(name))


_scorers = {}


def scorer(name, **cap):
    key = (name, tuple(sorted(cap.items())))
    if key not in _scorers:
        w = synth.WORKLOADS[name]
        cfg = config_for(w.shape, **cap)
        _scorers[key] = rm.Scorer(cfg, weights(name))
    return _scorers[key]


def gpu_scores(sc, ids, off, host=False):
    n = len(off) - 1
    if host:
        ids_h = torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).pin_memory()
        out_h = torch.empty(n, dtype=torch.float32).pin_memory()
        sc.score_host(ids_h, off, out_h)
        torch.cuda.synchronize()
        return out_h.numpy().astype(np.float64)
    ids_d = torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).cuda()
    out = torch.full((n,), float("nan"), dtype=torch.float32, device="cuda")
    sc.score(ids_d, off, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def oracle_scores(name, ids, off, sample):
    from oracle import scorer as O
    m = omodel(name)
    return np.array([O.score_one(m, ids[off[i]:off[i + 1]]) for i in sample])


@pytest.mark.parametrize("attn", [rm.ATTN_FUSED, rm.ATTN_MATERIALIZED], ids=["fused", "materialized"])
def test_tiny_encoder_all_sequences_match_golden_and_oracle(attn):
    w = synth.WORKLOADS["tiny-enc"]
    st = synth.make_stream(w)
    ids, off = synth.pack(st, np.arange(len(st.lengths)))
    got = gpu_scores(scorer("tiny-enc", max_batch_seqs=8, max_tokens=256, max_len=64,
                            attn_impl=attn), ids, off)
    ref = oracle_scores("tiny-enc", ids, off, range(len(off) - 1))
    gold = np.loadtxt(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_enc_scores.txt"))
    assert np.max(np.abs(ref - gold)) <= 1e-12
    assert np.max(np.abs(got - ref)) <= SCORE_ATOL, (got, ref)


@pytest.mark.parametrize("L", [64, 128, 256])
def test_tinybert_batch1(L):
    w = synth.WORKLOADS["tinybert-b1"]
    ids = synth.make_token_ids(L, w.shape.vocab, w.seed + L)
    off = np.array([0, L], dtype=np.int32)
    got = gpu_scores(scorer("tinybert-b1", max_batch_seqs=1, max_tokens=512, max_len=512), ids, off)
    ref = oracle_scores("tinybert-b1", ids, off, [0])
    assert abs(got[0] - ref[0]) <= SCORE_ATOL


def _dp_batches(name, n_req):
    w = synth.WORKLOADS[name]
    st = synth.make_stream(w, n_req)
    batch, _ = OS.schedule_dp(st.lengths, w.max_batch, OS.linear_cost(20000, 1))
    return st, batch


@pytest.mark.parametrize("name,n_req,which,n_sample,attn", [
    ("bert-base-len2-100", 2000, "last", 8, 0), ("bert-base-len2-100", 2000, "first", 8, 0),
    ("bert-base-len2-100", 2000, "last", 4, 1),
    ("bert-base-len5-500", 400, "last", 3, 0), ("bert-base-len5-500", 400, "last", 2, 1)])
def test_bert_base_dp_batch_sampled(name, n_req, which, n_sample, attn):
    w = synth.WORKLOADS[name]
    st, batch = _dp_batches(name, n_req)
    b = int(batch.max()) if which == "last" else 0
    idx = np.nonzero(batch == b)[0]
    ids, off = synth.pack(st, idx)
    sc = scorer(name, max_batch_seqs=w.max_batch, max_tokens=w.max_batch * w.len_hi,
                max_len=512, attn_impl=attn)
    got = gpu_scores(sc, ids, off)
    sample = np.linspace(0, len(idx) - 1, n_sample).astype(int)
    ref = oracle_scores(name, ids, off, sample)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got[sample] - ref)) <= SCORE_ATOL


def test_bench_launch_configuration_eight_fused_batches():
    """The call bench.py times: eight consecutive DP batches of the full
    10,000-request stream in one rm_score call (512 sequences, ~28k tokens),
    on a handle sized as bench.py sizes it; sampled sequences against the
    oracle, every score finite, and each sequence's score the same as when its
    own DP batch is scored alone."""
    name = "bert-base-len2-100"
    w = synth.WORKLOADS[name]
    st = synth.make_stream(w)
    cfg_sched = config_for(w.shape, max_len=100, sched_max_batch=w.max_batch, sched_c0=20000,
                           sched_c1=1)
    batch = rm.schedule(cfg_sched, st.lengths)
    idx = np.concatenate([np.nonzero(batch == b)[0] for b in range(80, 88)])
    ids, off = synth.pack(st, idx)
    sc = scorer(name, max_batch_seqs=8 * w.max_batch, max_tokens=8 * w.max_batch * 100, max_len=100)
    got = gpu_scores(sc, ids, off)
    assert len(idx) > 400 and np.all(np.isfinite(got))
    sample = np.linspace(0, len(idx) - 1, 6).astype(int)
    ref = oracle_scores(name, ids, off, sample)
    assert np.max(np.abs(got[sample] - ref)) <= SCORE_ATOL
    # the same requests as separate calls: the packed layout makes fusion invisible
    first = np.nonzero(batch == 80)[0]
    ids1, off1 = synth.pack(st, first)
    alone = gpu_scores(sc, ids1, off1)
    assert np.max(np.abs(alone - got[:len(first)])) <= 2e-3


@pytest.mark.parametrize("attn", [rm.ATTN_FUSED, rm.ATTN_MATERIALIZED], ids=["fused", "materialized"])
def test_bert_base_mixed_lengths_every_sequence(attn):
    """A ragged batch of every length class, all sequences checked."""
    name = "bert-base-len2-100"
    lens = np.array([1, 2, 3, 7, 8, 9, 63, 64, 65, 100, 127, 128, 129, 200, 511, 512])
    off = synth.offsets_from_lengths(lens)
    ids = synth.make_token_ids(int(off[-1]), 30522, 77)
    sc = scorer(name, max_batch_seqs=64, max_tokens=6400, max_len=512, attn_impl=attn)
    got = gpu_scores(sc, ids, off)
    ref = oracle_scores(name, ids, off, range(len(lens)))
    assert np.max(np.abs(got - ref)) <= SCORE_ATOL


@pytest.mark.parametrize("attn", [rm.ATTN_FUSED, rm.ATTN_MATERIALIZED], ids=["fused", "materialized"])
def test_decoder_small_shape_every_sequence(attn):
    """The pre-LN causal path on a small decoder (fast oracle), all sequences."""
    shape = synth.ModelShape(synth.DEC_PRELN, 3, 256, 4, 1024, 5000, 600, synth.W_BF16,
                             synth.GELU_ERF, 1e-5)
    flat = synth.make_weights(shape, 9)
    cfg = config_for(shape, max_batch_seqs=16, max_tokens=4096, max_len=600, attn_impl=attn)
    lens = np.array([1, 2, 65, 256, 300, 560, 17])
    off = synth.offsets_from_lengths(lens)
    ids = synth.make_token_ids(int(off[-1]), shape.vocab, 10)
    with rm.Scorer(cfg, flat) as sc:
        got = gpu_scores(sc, ids, off)
    from oracle import scorer as O
    m = oracle_model(shape, flat)
    ref = O.score_packed(m, ids, off)
    assert np.max(np.abs(got - ref)) <= SCORE_ATOL


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _report(label, err, lens):
    """One line per whole-batch check, so the GPU log records the error profile."""
    order = np.argsort(lens)
    print(f"\n{label}: max |gpu - oracle| = {err.max():.3e} over {len(err)} sequences; "
          f"8 shortest {err[order[:8]].max():.3e}, 8 longest {err[order[-8:]].max():.3e}")


@pytest.mark.slow
def test_gpt_1p3b_whole_batch_every_sequence():
    """Every sequence of a 64-sequence batch of the 1.3B-shape causal reward
    model (lengths U[256, 560], 24 pre-LN layers) against the fp64 oracle
    (scores written by tests/golden/make_golden.py; the shortest sequence is
    re-scored by the oracle here to tie the stored file to it)."""
    name = "gpt-1.3b-rm"
    w = synth.WORKLOADS[name]
    st = synth.make_stream(w)
    ids, off = synth.pack(st, np.arange(w.max_batch))
    gold = np.loadtxt(os.path.join(GOLDEN, "gpt_1p3b_rm_batch_scores.txt"))
    assert gold.shape == (w.max_batch,)
    sc = scorer(name, max_batch_seqs=64, max_tokens=64 * 560, max_len=560)
    got = gpu_scores(sc, ids, off)
    assert np.all(np.isfinite(got))
    lens = np.diff(off)
    err = np.abs(got - gold)
    _report(name, err, lens)
    assert err.max() <= SCORE_ATOL, (err.max(), int(np.argmax(err)), int(lens[np.argmax(err)]))
    i = int(np.argmin(lens))
    assert abs(oracle_scores(name, ids, off, [i])[0] - gold[i]) <= 1e-9


def test_bert_base_len5_500_longest_batch_every_sequence():
    """Every sequence of the last (longest) DP batch of the full 10,000-request
    lengths-5..500 stream (Bmax 32; rows up to 500 tokens) against the fp64
    oracle's stored scores, on both attention paths."""
    name = "bert-base-len5-500"
    w = synth.WORKLOADS[name]
    st = synth.make_stream(w)
    rows = np.loadtxt(os.path.join(GOLDEN, "bert_base_len5_500_longest_batch_scores.txt"))
    idx, gold = rows[:, 0].astype(np.int64), rows[:, 1]
    batch, _ = OS.schedule_dp(st.lengths, w.max_batch, OS.linear_cost(20000, 1))
    assert np.array_equal(np.nonzero(batch == batch.max())[0], idx)
    ids, off = synth.pack(st, idx)
    lens = np.diff(off)
    for attn in (rm.ATTN_FUSED, rm.ATTN_MATERIALIZED):
        sc = scorer(name, max_batch_seqs=w.max_batch, max_tokens=w.max_batch * w.len_hi, max_len=512,
                    attn_impl=attn)
        got = gpu_scores(sc, ids, off)
        err = np.abs(got - gold)
        _report(f"{name} attn_impl={attn}", err, lens)
        assert err.max() <= SCORE_ATOL, (attn, err.max(), int(lens[np.argmax(err)]))
    i = int(np.argmax(lens))
    assert abs(oracle_scores(name, ids, off, [i])[0] - gold[i]) <= 1e-9


# --- edge cases -----------------------------------------------------------------------

def test_single_token_and_max_len_sequences():
    name = "tiny-enc"
    sc = scorer(name, max_batch_seqs=8, max_tokens=256, max_len=64)
    for lens in ([1], [64], [1, 64, 1], [64] * 4):
        lens = np.array(lens)
        off = synth.offsets_from_lengths(lens)
        ids = synth.make_token_ids(int(off[-1]), 1000, len(lens))
        got = gpu_scores(sc, ids, off)
        ref = oracle_scores(name, ids, off, range(len(lens)))
        assert np.max(np.abs(got - ref)) <= SCORE_ATOL


def test_host_entry_point_equals_device_entry_point_and_is_deterministic():
    name = "bert-base-len2-100"
    st, batch = _dp_batches(name, 500)
    idx = np.nonzero(batch == 3)[0]
    ids, off = synth.pack(st, idx)
    sc = scorer(name, max_batch_seqs=64, max_tokens=6400, max_len=512)
    a = gpu_scores(sc, ids, off)
    b = gpu_scores(sc, ids, off, host=True)
    c = gpu_scores(sc, ids, off)
    assert np.array_equal(a, b) and np.array_equal(a, c)


def test_arena_does_not_grow_after_warmup():
    name = "bert-base-len2-100"
    sc = scorer(name, max_batch_seqs=64, max_tokens=6400, max_len=512)
    st, batch = _dp_batches(name, 1000)
    for b in range(int(batch.max()) + 1):
        ids, off = synth.pack(st, np.nonzero(batch == b)[0])
        gpu_scores(sc, ids, off)
    reserved, used, nbuckets = sc.arena_stats()
    assert used <= reserved and nbuckets >= 1
    for b in range(int(batch.max()) + 1):
        ids, off = synth.pack(st, np.nonzero(batch == b)[0])
        gpu_scores(sc, ids, off)
    assert tuple(sc.arena_stats()) == (reserved, used, nbuckets)


def test_out_of_range_ids_are_clamped_and_counted():
    sc = rm.Scorer(config_for(synth.TINY, max_batch_seqs=4, max_tokens=64, max_len=64),
                   weights("tiny-enc"))
    ids = np.array([5, 999, 1000, -1, 7], dtype=np.int32)
    off = np.array([0, 2, 5], dtype=np.int32)
    got = gpu_scores(sc, ids, off)
    ref = oracle_scores("tiny-enc", np.clip(ids, 0, 999), off, [0, 1])
    assert np.max(np.abs(got - ref)) <= SCORE_ATOL
    clamped, timeouts = sc.device_error()
    assert clamped == 2 and timeouts == 0
    sc.close()


def test_invalid_calls_are_rejected_before_any_work():
    sc = scorer("tiny-enc", max_batch_seqs=8, max_tokens=256, max_len=64)
    ids = torch.zeros(300, dtype=torch.int32, device="cuda")
    out = torch.zeros(16, dtype=torch.float32, device="cuda")
    cases = [
        (np.array([0], dtype=np.int32), rm.RM_E_INVAL),             # n = 0
        (np.array([1, 5], dtype=np.int32), rm.RM_E_INVAL),          # offsets[0] != 0
        (np.array([0, 5, 5], dtype=np.int32), rm.RM_E_INVAL),       # empty sequence
        (np.array([0, 5, 3], dtype=np.int32), rm.RM_E_INVAL),       # decreasing
        (np.array([0, 65], dtype=np.int32), rm.RM_E_RANGE),         # > max_len
        (np.arange(0, 10 * 9, 9, dtype=np.int32), rm.RM_E_RANGE),   # 9 > max_batch_seqs
        (np.array([0, 64, 128, 192, 256, 300], dtype=np.int32), rm.RM_E_RANGE),  # > max_tokens
    ]
    for off, code in cases:
        with pytest.raises(rm.RmError) as e:
            sc.score(ids, off, out)
        assert e.value.code == code, (off, e.value)
    assert sc.device_error()[1] == 0


def test_handle_schedule_matches_oracle():
    w = synth.WORKLOADS["bert-base-len2-100"]
    sc = scorer("bert-base-len2-100", max_batch_seqs=64, max_tokens=6400, max_len=512)
    lengths = synth.make_stream(w).lengths
    ref, _ = OS.schedule_dp(lengths, 64, OS.linear_cost(0, 1))
    assert np.array_equal(sc.schedule(lengths), ref)


def test_shared_handles_on_two_streams_match_one_handle():
    name = "bert-base-len2-100"
    w = synth.WORKLOADS[name]
    st, batch = _dp_batches(name, 800)
    base = rm.Scorer(config_for(w.shape, max_batch_seqs=64, max_tokens=6400, max_len=512),
                     weights(name))
    other = base.shared()
    batches = [np.nonzero(batch == b)[0] for b in range(int(batch.max()) + 1)]
    packed = [synth.pack(st, idx) for idx in batches]
    ref = [gpu_scores(base, ids, off) for ids, off in packed]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    handles = [base, other]
    outs = []
    ids_d = [torch.from_numpy(ids).cuda() for ids, _ in packed]
    torch.cuda.synchronize()
    for k, (ids, off) in enumerate(packed):
        o = torch.full((len(off) - 1,), float("nan"), dtype=torch.float32, device="cuda")
        handles[k % 2].score(ids_d[k], off, o, streams[k % 2])
        outs.append(o)
    torch.cuda.synchronize()
    for o, r in zip(outs, ref):
        assert np.array_equal(o.cpu().numpy().astype(np.float64), r)
    # the weights outlive the handle that uploaded them
    base.close()
    ids, off = packed[0]
    assert np.array_equal(gpu_scores(other, ids, off), ref[0])
    other.close()
