"""fp64 forward pass of the compact transformer scorer (TEST INFRASTRUCTURE ONLY).

What is computed, and where it comes from:

* The encoder scorer is a compact BERT/TinyBERT-style transformer encoder
  (TinyBERT on the SambaNova blog "Breakthrough efficiency in NLP model
  deployment", first section; the transformer encoder served in
  "TurboTransformers: An Efficient GPU Serving System For Transformer Models",
  abstract).  Post-LN layers: x = LN1(x + MHA(x)), x = LN2(x + FFN(x)).
* The reward model is a GPT-style decoder initialised from a supervised
  baseline with a scalar head added ("Learning to summarize from human
  feedback" summary, method section).  Pre-LN causal layers:
  x = x + MHA_causal(LN1(x)), x = x + FFN(LN2(x)), final LN_f, head on the
  last token.  The reward normalisation of that section (reference summaries
  average zero) is a constant shift and is absorbed into the head bias b_r.
* Softmax and LayerNorm are the two "batch reduction" operations that the
  TurboTransformers abstract names as the hot spots besides the GEMMs, and
  variable-length input is served without padding (same abstract and the
  proposed-method section).  Each sequence is therefore computed on its own
  (``score_packed``); ``score_padded`` is the padded-and-masked formulation
  that must give the same result.

Readings where the pages are silent (each also listed in the design notes):
no token-type embeddings; no tanh pooler (the head reads token 0 of the
encoder output directly); GELU is the erf form unless the tanh flag is set;
LayerNorm uses the biased variance; epsilon is a model parameter.

Everything here is plain numpy in float64.  A matmul (``@``) is the only
library primitive used as a step; erf comes from scipy.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import numpy as np
from scipy.special import erf

ENC_POSTLN = 0
DEC_PRELN = 1
GELU_ERF = 0
GELU_TANH = 1


@dataclasses.dataclass
class OracleModel:
    arch: int
    n_layers: int
    hidden: int
    n_heads: int
    ffn: int
    vocab: int
    max_pos: int
    gelu: int
    ln_eps: float
    p: Dict[str, np.ndarray]          # float64 tensors by name
    layers: List[Dict[str, np.ndarray]]


def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    # a bf16 value is the upper half of an fp32 bit pattern
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def unpack_weights(flat, arch, n_layers, hidden, n_heads, ffn, vocab, max_pos,
                   weight_dtype, gelu=GELU_ERF, ln_eps=1e-12) -> OracleModel:
    """Parse the flat weight buffer in the order the C ABI documents.

    Order: word embeddings [V][H], position embeddings [P][H], (encoder:
    embedding LN gain, bias), then per layer W_qkv[3H][H], b_qkv[3H],
    W_o[H][H], b_o[H], LN1 gain, bias, W_1[F][H], b_1[F], W_2[H][F], b_2[H],
    LN2 gain, bias; (decoder: final LN gain, bias); head w_r[H], b_r[1].
    weight_dtype 0 = float32 values, 1 = bf16 bit patterns (uint16).
    """
    flat = np.asarray(flat)
    vals = _bf16_bits_to_f64(flat) if weight_dtype == 1 else flat.astype(np.float64)
    H, F = hidden, ffn
    pos = 0

    def take(*shape):
        nonlocal pos
        n = int(np.prod(shape))
        t = vals[pos:pos + n].reshape(shape)
        pos += n
        return t

    p = {"emb_word": take(vocab, H), "emb_pos": take(max_pos, H)}
    if arch == ENC_POSTLN:
        p["ln_emb_g"] = take(H)
        p["ln_emb_b"] = take(H)
    layers = []
    for _ in range(n_layers):
        lw = {}
        lw["w_qkv"] = take(3 * H, H)
        lw["b_qkv"] = take(3 * H)
        lw["w_o"] = take(H, H)
        lw["b_o"] = take(H)
        lw["ln1_g"] = take(H)
        lw["ln1_b"] = take(H)
        lw["w_1"] = take(F, H)
        lw["b_1"] = take(F)
        lw["w_2"] = take(H, F)
        lw["b_2"] = take(H)
        lw["ln2_g"] = take(H)
        lw["ln2_b"] = take(H)
        layers.append(lw)
    if arch == DEC_PRELN:
        p["lnf_g"] = take(H)
        p["lnf_b"] = take(H)
    p["w_r"] = take(H)
    p["b_r"] = take(1)
    if pos != vals.size:
        raise ValueError(f"weight buffer holds {vals.size} values, layout needs {pos}")
    return OracleModel(arch, n_layers, hidden, n_heads, ffn, vocab, max_pos, gelu,
                       float(ln_eps), p, layers)


# ---------------------------------------------------------------------------
# The two batch reductions (TurboTransformers abstract and proposed-method
# section: Softmax and LayerNorm as parallel batch reductions).
# ---------------------------------------------------------------------------

def layer_norm(y: np.ndarray, gain: np.ndarray, bias: np.ndarray, eps: float) -> np.ndarray:
    """LN over the last axis: gain * (y - mean) / sqrt(var + eps) + bias, biased var."""
    mu = y.mean(axis=-1, keepdims=True)
    var = ((y - mu) ** 2).mean(axis=-1, keepdims=True)
    return gain * (y - mu) / np.sqrt(var + eps) + bias


def softmax_masked(s: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    """Row softmax over the allowed entries only; disallowed entries are exactly 0.

    p_c = exp(s_c - max_allowed) / sum_allowed exp(s_c' - max_allowed).
    Every row must allow at least one entry.
    """
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    e = np.where(allowed, np.exp(s - m), 0.0)
    return e / e.sum(axis=-1, keepdims=True)


def linear(x: np.ndarray, w: np.ndarray, b) -> np.ndarray:
    """x W^T + b with W stored [out][in] (b may be None)."""
    y = x @ w.T
    return y if b is None else y + b


def gelu(u: np.ndarray, kind: int = GELU_ERF) -> np.ndarray:
    """GELU: u * Phi(u) with the normal CDF Phi (erf form), or the tanh approximation."""
    if kind == GELU_ERF:
        return u * 0.5 * (1.0 + erf(u / np.sqrt(2.0)))
    c = np.sqrt(2.0 / np.pi)
    return 0.5 * u * (1.0 + np.tanh(c * (u + 0.044715 * u ** 3)))


# ---------------------------------------------------------------------------
# One sequence, padding-free.
# ---------------------------------------------------------------------------

def embed(m: OracleModel, ids: np.ndarray) -> np.ndarray:
    """x_t = E_word[id_t] + E_pos[t] for t = 0..L-1 (encoder: then the embedding LN)."""
    L = len(ids)
    x = m.p["emb_word"][np.asarray(ids, dtype=np.int64)] + m.p["emb_pos"][:L]
    if m.arch == ENC_POSTLN:
        x = layer_norm(x, m.p["ln_emb_g"], m.p["ln_emb_b"], m.ln_eps)
    return x


def attention_probs(q: np.ndarray, k: np.ndarray, causal: bool) -> np.ndarray:
    """P = softmax over keys of q_r . k_c / sqrt(d), keys c <= r when causal."""
    d = q.shape[-1]
    s = (q @ k.T) / np.sqrt(d)
    L = q.shape[0]
    allowed = np.ones((L, L), dtype=bool)
    if causal:
        allowed = np.tril(allowed)
    return softmax_masked(s, allowed)


def mha(x: np.ndarray, lw: Dict[str, np.ndarray], n_heads: int, causal: bool) -> np.ndarray:
    """Multi-head self-attention of one sequence x[L][H].

    q, k, v = x W_q^T + b_q, ...; per head j the columns j*d..j*d+d-1;
    o = concat_j P_j v_j; output o W_o^T + b_o.
    """
    L, H = x.shape
    d = H // n_heads
    qkv = linear(x, lw["w_qkv"], lw["b_qkv"])
    q, k, v = qkv[:, :H], qkv[:, H:2 * H], qkv[:, 2 * H:]
    o = np.empty((L, H))
    for j in range(n_heads):
        cols = slice(j * d, (j + 1) * d)
        pj = attention_probs(q[:, cols], k[:, cols], causal)
        o[:, cols] = pj @ v[:, cols]
    return linear(o, lw["w_o"], lw["b_o"])


def ffn(x: np.ndarray, lw: Dict[str, np.ndarray], kind: int) -> np.ndarray:
    """W_2 GELU(W_1 x + b_1) + b_2, row-wise."""
    return linear(gelu(linear(x, lw["w_1"], lw["b_1"]), kind), lw["w_2"], lw["b_2"])


def encoder_layer(x, lw, m: OracleModel):
    """Post-LN encoder layer: x = LN1(x + MHA(x)); x = LN2(x + FFN(x))."""
    x = layer_norm(x + mha(x, lw, m.n_heads, causal=False), lw["ln1_g"], lw["ln1_b"], m.ln_eps)
    return layer_norm(x + ffn(x, lw, m.gelu), lw["ln2_g"], lw["ln2_b"], m.ln_eps)


def decoder_layer(x, lw, m: OracleModel):
    """Pre-LN causal decoder layer: x += MHA_causal(LN1(x)); x += FFN(LN2(x))."""
    x = x + mha(layer_norm(x, lw["ln1_g"], lw["ln1_b"], m.ln_eps), lw, m.n_heads, causal=True)
    return x + ffn(layer_norm(x, lw["ln2_g"], lw["ln2_b"], m.ln_eps), lw, m.gelu)


def hidden_states(m: OracleModel, ids: np.ndarray) -> np.ndarray:
    """Final hidden states [L][H] of one sequence (decoder: before LN_f)."""
    x = embed(m, ids)
    for lw in m.layers:
        x = encoder_layer(x, lw, m) if m.arch == ENC_POSTLN else decoder_layer(x, lw, m)
    return x


def head(m: OracleModel, h: np.ndarray) -> float:
    """Scalar head: encoder w_r . h_0 + b_r; decoder w_r . LN_f(h_{L-1}) + b_r."""
    if m.arch == ENC_POSTLN:
        z = h[0]
    else:
        z = layer_norm(h[-1], m.p["lnf_g"], m.p["lnf_b"], m.ln_eps)
    return float(z @ m.p["w_r"] + m.p["b_r"][0])


def score_one(m: OracleModel, ids: np.ndarray) -> float:
    return head(m, hidden_states(m, ids))


def score_packed(m: OracleModel, ids: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    """Scores of every sequence i = ids[offsets[i]:offsets[i+1]], each on its own."""
    n = len(offsets) - 1
    return np.array([score_one(m, ids[offsets[i]:offsets[i + 1]]) for i in range(n)])


# ---------------------------------------------------------------------------
# Padded-and-masked formulation (the fixed-length batch that the
# TurboTransformers proposed-method section avoids); used only to check that
# padding-free equals padded-and-masked.
# ---------------------------------------------------------------------------

def score_padded(m: OracleModel, ids: np.ndarray, offsets: np.ndarray, pad_id: int = 0) -> np.ndarray:
    n = len(offsets) - 1
    lens = np.diff(offsets)
    Lmax = int(lens.max())
    H, nh = m.hidden, m.n_heads
    d = H // nh
    tok = np.full((n, Lmax), pad_id, dtype=np.int64)
    for i in range(n):
        tok[i, :lens[i]] = ids[offsets[i]:offsets[i + 1]]
    key_ok = np.arange(Lmax)[None, :] < lens[:, None]                  # [n][Lmax]
    x = m.p["emb_word"][tok] + m.p["emb_pos"][:Lmax][None]
    if m.arch == ENC_POSTLN:
        x = layer_norm(x, m.p["ln_emb_g"], m.p["ln_emb_b"], m.ln_eps)
    causal = m.arch == DEC_PRELN
    allowed = np.broadcast_to(key_ok[:, None, None, :], (n, nh, Lmax, Lmax)).copy()
    if causal:
        allowed &= np.tril(np.ones((Lmax, Lmax), dtype=bool))[None, None]
    # padded query rows still need one allowed key; they are discarded anyway
    allowed[..., 0] = True

    def batched_mha(z, lw):
        qkv = z @ lw["w_qkv"].T + lw["b_qkv"]
        q = qkv[..., :H].reshape(n, Lmax, nh, d).transpose(0, 2, 1, 3)
        k = qkv[..., H:2 * H].reshape(n, Lmax, nh, d).transpose(0, 2, 1, 3)
        v = qkv[..., 2 * H:].reshape(n, Lmax, nh, d).transpose(0, 2, 1, 3)
        s = q @ k.transpose(0, 1, 3, 2) / np.sqrt(d)
        pr = softmax_masked(s, allowed)
        o = (pr @ v).transpose(0, 2, 1, 3).reshape(n, Lmax, H)
        return o @ lw["w_o"].T + lw["b_o"]

    for lw in m.layers:
        if m.arch == ENC_POSTLN:
            x = layer_norm(x + batched_mha(x, lw), lw["ln1_g"], lw["ln1_b"], m.ln_eps)
            x = layer_norm(x + ffn(x, lw, m.gelu), lw["ln2_g"], lw["ln2_b"], m.ln_eps)
        else:
            x = x + batched_mha(layer_norm(x, lw["ln1_g"], lw["ln1_b"], m.ln_eps), lw)
            x = x + ffn(layer_norm(x, lw["ln2_g"], lw["ln2_b"], m.ln_eps), lw, m.gelu)
    out = np.empty(n)
    for i in range(n):
        out[i] = head(m, x[i, :lens[i]])
    return out
