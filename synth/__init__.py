"""Seeded synthetic inputs for the transformer scorer.

This module is the only code that both the CUDA path's harness (tests, bench)
and the fp64 oracle's tests consume.  It holds no arithmetic of the scoring
method itself: it only draws random numbers and lays them out in the flat
weight format that the C ABI documents (``include/rm.h``), plus token ids,
lengths and arrival times for request streams.

Workload shapes follow the pages:
  * lengths 2..100 and 5..500 for the TurboTransformers serving study
    ("TurboTransformers: An Efficient GPU Serving System For Transformer
    Models" review, main results);
  * fixed lengths 64/128/256 at batch 1 for the TinyBERT latency study
    (SambaNova blog, Figure 3);
  * a 1.3B GPT-style reward model with a scalar head on a post plus a short
    summary ("Learning to summarize from human feedback" summary, compute
    setup and method sections).
Weights are drawn N(0, 0.02); LayerNorm gains are 1 + N(0, 0.02) so every
fused term of the forward pass is observable.
"""
from __future__ import annotations

import dataclasses
from typing import List, Tuple

import numpy as np

ENC_POSTLN = 0
DEC_PRELN = 1
W_F32 = 0
W_BF16 = 1
GELU_ERF = 0
GELU_TANH = 1


@dataclasses.dataclass(frozen=True)
class ModelShape:
    arch: int
    n_layers: int
    hidden: int
    n_heads: int
    ffn: int
    vocab: int
    max_pos: int
    weight_dtype: int
    gelu: int = GELU_ERF
    ln_eps: float = 1e-12

    @property
    def head_dim(self) -> int:
        return self.hidden // self.n_heads


@dataclasses.dataclass(frozen=True)
class Workload:
    """A named synthetic workload: model shape plus request-stream recipe."""
    name: str
    shape: ModelShape
    seed: int
    len_lo: int
    len_hi: int
    n_requests: int
    max_batch: int
    fixed_lengths: Tuple[int, ...] = ()


TINY = ModelShape(ENC_POSTLN, 2, 128, 2, 512, 1000, 64, W_F32, GELU_ERF, 1e-12)
TINYBERT = ModelShape(ENC_POSTLN, 4, 312, 12, 1200, 30522, 512, W_BF16, GELU_ERF, 1e-12)
BERT_BASE = ModelShape(ENC_POSTLN, 12, 768, 12, 3072, 30522, 512, W_BF16, GELU_ERF, 1e-12)
GPT_1P3B = ModelShape(DEC_PRELN, 24, 2048, 16, 8192, 50257, 2048, W_BF16, GELU_ERF, 1e-5)

WORKLOADS = {
    "tiny-enc": Workload("tiny-enc", TINY, 0, 8, 32, 4, 4),
    "tinybert-b1": Workload("tinybert-b1", TINYBERT, 1, 64, 256, 1, 1, (64, 128, 256)),
    "bert-base-len2-100": Workload("bert-base-len2-100", BERT_BASE, 2, 2, 100, 10000, 64),
    "bert-base-len5-500": Workload("bert-base-len5-500", BERT_BASE, 3, 5, 500, 10000, 32),
    "gpt-1.3b-rm": Workload("gpt-1.3b-rm", GPT_1P3B, 4, 256, 560, 64, 64),
}


@dataclasses.dataclass(frozen=True)
class PrefixWorkload:
    """Best-of-N scoring: n_groups prefixes (posts), each followed by n_cand
    candidates (summaries), lengths uniform on the stated integer ranges."""
    name: str
    shape: ModelShape
    seed: int
    n_groups: int
    n_cand: int
    prefix_lo: int
    prefix_hi: int
    cand_lo: int
    cand_hi: int
    weight_seed: int


# TL;DR-shaped best-of-8: posts + summaries of at most 48 tokens, totals within
# the 256..560 range of the gpt-1.3b-rm stream
PREFIX_WORKLOADS = {
    # the same weights as gpt-1.3b-rm (seed 4), its own requests (seed 5)
    "gpt-1.3b-best-of-8": PrefixWorkload("gpt-1.3b-best-of-8", GPT_1P3B, 5, 8, 8, 208, 512, 24, 48, 4),
}


def make_prefix_groups(w: PrefixWorkload, seed_offset: int = 0):
    """(ids, prefix_len, n_cand, cand_len) in the packed shared-prefix layout:
    per group its prefix, then its candidates."""
    seed = w.seed + seed_offset
    prefix_len = make_lengths(w.n_groups, w.prefix_lo, w.prefix_hi, seed)
    cand_len = make_lengths(w.n_groups * w.n_cand, w.cand_lo, w.cand_hi, seed + 7919)
    n_cand = np.full(w.n_groups, w.n_cand, dtype=np.int32)
    total = int(prefix_len.astype(np.int64).sum() + cand_len.astype(np.int64).sum())
    ids = make_token_ids(total, w.shape.vocab, seed)
    return ids, prefix_len, n_cand, cand_len


def weight_segments(s: ModelShape) -> List[Tuple[str, Tuple[int, ...], str]]:
    """(name, shape, kind) of every tensor in flat-buffer order.

    kind is 'normal' (N(0, 0.02)) or 'gain' (1 + N(0, 0.02)).
    Linear weights are [out][in] row-major; Q, K, V rows are stacked in that
    order, head j of each owning rows j*d .. j*d+d-1.
    """
    H, F = s.hidden, s.ffn
    seg = [("emb_word", (s.vocab, H), "normal"), ("emb_pos", (s.max_pos, H), "normal")]
    if s.arch == ENC_POSTLN:
        seg += [("ln_emb_g", (H,), "gain"), ("ln_emb_b", (H,), "normal")]
    for l in range(s.n_layers):
        p = f"l{l}."
        seg += [
            (p + "w_qkv", (3 * H, H), "normal"), (p + "b_qkv", (3 * H,), "normal"),
            (p + "w_o", (H, H), "normal"), (p + "b_o", (H,), "normal"),
            (p + "ln1_g", (H,), "gain"), (p + "ln1_b", (H,), "normal"),
            (p + "w_1", (F, H), "normal"), (p + "b_1", (F,), "normal"),
            (p + "w_2", (H, F), "normal"), (p + "b_2", (H,), "normal"),
            (p + "ln2_g", (H,), "gain"), (p + "ln2_b", (H,), "normal"),
        ]
    if s.arch == DEC_PRELN:
        seg += [("lnf_g", (H,), "gain"), ("lnf_b", (H,), "normal")]
    seg += [("w_r", (H,), "normal"), ("b_r", (1,), "normal")]
    return seg


def n_weight_elems(s: ModelShape) -> int:
    return int(sum(int(np.prod(shp)) for _, shp, _ in weight_segments(s)))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = b + (((b >> 16) & 1) + 0x7FFF)
    return (b >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def make_weights(s: ModelShape, seed: int, std: float = 0.02) -> np.ndarray:
    """Flat weight buffer: float32 for W_F32, uint16 bf16 bits for W_BF16."""
    rng = np.random.default_rng([seed, 0x5EED])
    out = np.empty(n_weight_elems(s), dtype=np.float32)
    pos = 0
    for _, shp, kind in weight_segments(s):
        n = int(np.prod(shp))
        v = out[pos:pos + n]
        rng.standard_normal(n, dtype=np.float32, out=v)
        v *= np.float32(std)
        if kind == "gain":
            v += np.float32(1.0)
        pos += n
    if s.weight_dtype == W_BF16:
        return f32_to_bf16_bits(out)
    return out


def make_lengths(n: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """n lengths uniform on the integers lo..hi inclusive (int32)."""
    rng = np.random.default_rng([seed, 0x1E9])
    return rng.integers(lo, hi + 1, size=n, dtype=np.int64).astype(np.int32)


def make_token_ids(total: int, vocab: int, seed: int) -> np.ndarray:
    """total token ids uniform on 0..vocab-1 (int32)."""
    rng = np.random.default_rng([seed, 0x70C])
    return rng.integers(0, vocab, size=total, dtype=np.int64).astype(np.int32)


def make_arrivals(n: int, rate_per_s: float, seed: int) -> np.ndarray:
    """Poisson arrival times (seconds, float64) with exponential gaps."""
    rng = np.random.default_rng([seed, 0xA77])
    return np.cumsum(rng.exponential(1.0 / rate_per_s, size=n))


def offsets_from_lengths(lengths: np.ndarray) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, dtype=np.int32)
    off[1:] =np.cumsum(np.asarray(lengths, dtype=np.int64)).astype(np.int32)
    return off


@dataclasses.dataclass
class Stream:
    lengths: np.ndarray      # int32[n]
    ids: np.ndarray          # int32[sum(lengths)], request i at ids[starts[i]:starts[i]+lengths[i]]
    starts: np.ndarray       # int64[n]


def make_stream(w: Workload, n: int | None = None) -> Stream:
    """The seeded request stream of a workload (first n requests if given).

    The stream is a property of the seed, so a prefix of the stream is the
    same whatever n is requested.
    """
    n_all = w.n_requests
    if w.fixed_lengths:
        lengths = np.array(w.fixed_lengths, dtype=np.int32)
        n_all = len(lengths)
    else:
        lengths = make_lengths(n_all, w.len_lo, w.len_hi, w.seed)
    starts = np.zeros(n_all, dtype=np.int64)
    starts[1:] = np.cumsum(lengths[:-1].astype(np.int64))
    ids = make_token_ids(int(lengths.astype(np.int64).sum()), w.shape.vocab, w.seed)
    if n is not None:
        lengths = lengths[:n]
        starts = starts[:n]
        ids = ids[: int(starts[-1] + lengths[-1])] if n > 0 else ids[:0]
    return Stream(lengths=lengths, ids=ids, starts=starts)


def pack(stream: Stream, idx: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Gather requests idx of a stream into packed ids and seq offsets."""
    idx = np.asarray(idx, dtype=np.int64)
    lens = stream.lengths[idx]
    off = offsets_from_lengths(lens)
    ids = np.empty(int(off[-1]), dtype=np.int32)
    for k, i in enumerate(idx):
        ids[off[k]:off[k + 1]] = stream.ids[stream.starts[i]:stream.starts[i] + stream.lengths[i]]
    return ids, off
