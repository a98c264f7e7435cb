"""Pins for the oracle's encoder and decoder forward passes.

The oracle is checked against independent implementations of the same
textbook models in float64 (torch's TransformerEncoderLayer, the
``transformers`` BertModel and GPT2Model), against closed forms, and against
invariants the architecture fixes.  Weights are drawn with a larger spread
than the workloads use so that attention is far from uniform and every term
moves the result.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import scorer as O

ENC = synth.ModelShape(synth.ENC_POSTLN, 2, 64, 4, 160, 97, 40, synth.W_F32, synth.GELU_ERF, 1e-12)
DEC = synth.ModelShape(synth.DEC_PRELN, 2, 64, 4, 160, 97, 40, synth.W_F32, synth.GELU_ERF, 1e-5)


def model(shape, seed=11, std=0.15, flat=None):
    if flat is None:
        flat = synth.make_weights(shape, seed, std=std)
    return O.unpack_weights(flat, shape.arch, shape.n_layers, shape.hidden, shape.n_heads,
                            shape.ffn, shape.vocab, shape.max_pos, shape.weight_dtype,
                            shape.gelu, shape.ln_eps)


def ids_for(shape, L, seed=3):
    return np.random.default_rng(seed).integers(0, shape.vocab, size=L)


# --- layout --------------------------------------------------------------------

def test_unpack_follows_documented_order():
    flat = np.arange(synth.n_weight_elems(ENC), dtype=np.float32)
    m = model(ENC, flat=flat)
    H, F, V, P = ENC.hidden, ENC.ffn, ENC.vocab, ENC.max_pos
    assert m.p["emb_word"][0, 0] == 0 and m.p["emb_word"][1, 0] == H
    assert m.p["emb_pos"][0, 0] == V * H
    base = V * H + P * H + 2 * H
    assert m.layers[0]["w_qkv"][0, 1] == base + 1
    assert m.layers[0]["w_qkv"][1, 0] == base + H          # [out][in], row-major
    assert m.layers[0]["b_qkv"][0] == base + 3 * H * H
    assert m.p["b_r"][0] == flat[-1]
    assert m.p["w_r"][0] == flat.size - 1 - H
    with pytest.raises(ValueError):
        model(ENC, flat=flat[:-1])


def test_unpack_bf16_bits():
    shape = dataclasses.replace(ENC, weight_dtype=synth.W_BF16)
    flat = synth.make_weights(shape, 5)
    m = model(shape, flat=flat)
    assert m.p["emb_word"][0, 0] == float(synth.bf16_bits_to_f32(flat[:1])[0])


# --- one layer against torch -----------------------------------------------------

def _torch_layer(shape, lw, norm_first):
    layer = torch.nn.TransformerEncoderLayer(
        d_model=shape.hidden, nhead=shape.n_heads, dim_feedforward=shape.ffn, dropout=0.0,
        activation="gelu", layer_norm_eps=shape.ln_eps, batch_first=True, norm_first=norm_first,
        dtype=torch.float64)
    with torch.no_grad():
        layer.self_attn.in_proj_weight.copy_(torch.from_numpy(lw["w_qkv"]))
        layer.self_attn.in_proj_bias.copy_(torch.from_numpy(lw["b_qkv"]))
        layer.self_attn.out_proj.weight.copy_(torch.from_numpy(lw["w_o"]))
        layer.self_attn.out_proj.bias.copy_(torch.from_numpy(lw["b_o"]))
        layer.linear1.weight.copy_(torch.from_numpy(lw["w_1"]))
        layer.linear1.bias.copy_(torch.from_numpy(lw["b_1"]))
        layer.linear2.weight.copy_(torch.from_numpy(lw["w_2"]))
        layer.linear2.bias.copy_(torch.from_numpy(lw["b_2"]))
        layer.norm1.weight.copy_(torch.from_numpy(lw["ln1_g"]))
        layer.norm1.bias.copy_(torch.from_numpy(lw["ln1_b"]))
        layer.norm2.weight.copy_(torch.from_numpy(lw["ln2_g"]))
        layer.norm2.bias.copy_(torch.from_numpy(lw["ln2_b"]))
    return layer.train(False)


def test_encoder_layer_matches_torch_post_ln_layer():
    m = model(ENC)
    x = np.random.default_rng(1).normal(size=(23, ENC.hidden))
    ours = O.encoder_layer(x, m.layers[0], m)
    layer = _torch_layer(ENC, m.layers[0], norm_first=False)
    with torch.no_grad():
        ref = layer(torch.from_numpy(x)[None])[0].numpy()
    assert np.max(np.abs(ours - ref)) <= 1e-10


def test_decoder_layer_matches_torch_pre_ln_causal_layer():
    m = model(DEC)
    L = 19
    x = np.random.default_rng(2).normal(size=(L, DEC.hidden))
    ours = O.decoder_layer(x, m.layers[1], m)
    layer = _torch_layer(DEC, m.layers[1], norm_first=True)
    mask = torch.triu(torch.ones(L, L, dtype=torch.bool), diagonal=1)   # True = masked
    with torch.no_grad():
        ref = layer(torch.from_numpy(x)[None], src_mask=mask)[0].numpy()
    assert np.max(np.abs(ours - ref)) <= 1e-10


# --- whole models against transformers ------------------------------------------------

def test_encoder_scores_match_bert_model():
    from transformers import BertConfig, BertModel
    m = model(ENC)
    cfg = BertConfig(vocab_size=ENC.vocab, hidden_size=ENC.hidden, num_hidden_layers=ENC.n_layers,
                     num_attention_heads=ENC.n_heads, intermediate_size=ENC.ffn, hidden_act="gelu",
                     hidden_dropout_prob=0.0, attention_probs_dropout_prob=0.0,
                     max_position_embeddings=ENC.max_pos, type_vocab_size=1,
                     layer_norm_eps=ENC.ln_eps, attn_implementation="eager")
    bert = BertModel(cfg, add_pooling_layer=False).to(torch.float64).train(False)
    H = ENC.hidden
    sd = {"embeddings.word_embeddings.weight": m.p["emb_word"],
          "embeddings.position_embeddings.weight": m.p["emb_pos"],
          "embeddings.token_type_embeddings.weight": np.zeros((1, H)),
          "embeddings.LayerNorm.weight": m.p["ln_emb_g"], "embeddings.LayerNorm.bias": m.p["ln_emb_b"]}
    for l, lw in enumerate(m.layers):
        p = f"encoder.layer.{l}."
        for j, nm in enumerate(("query", "key", "value")):
            sd[p + f"attention.self.{nm}.weight"] = lw["w_qkv"][j * H:(j + 1) * H]
            sd[p + f"attention.self.{nm}.bias"] = lw["b_qkv"][j * H:(j + 1) * H]
        sd[p + "attention.output.dense.weight"] = lw["w_o"]
        sd[p + "attention.output.dense.bias"] = lw["b_o"]
        sd[p + "attention.output.LayerNorm.weight"] = lw["ln1_g"]
        sd[p + "attention.output.LayerNorm.bias"] = lw["ln1_b"]
        sd[p + "intermediate.dense.weight"] = lw["w_1"]
        sd[p + "intermediate.dense.bias"] = lw["b_1"]
        sd[p + "output.dense.weight"] = lw["w_2"]
        sd[p + "output.dense.bias"] = lw["b_2"]
        sd[p + "output.LayerNorm.weight"] = lw["ln2_g"]
        sd[p + "output.LayerNorm.bias"] = lw["ln2_b"]
    bert.load_state_dict({k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in sd.items()},
                         strict=False)
    lens = np.array([1, 7, 23, 40, 2])
    off = synth.offsets_from_lengths(lens)
    ids = ids_for(ENC, int(off[-1]), seed=9)
    ours = O.score_packed(m, ids, off)
    tok = torch.zeros(len(lens), lens.max(), dtype=torch.long)
    att = torch.zeros(len(lens), lens.max(), dtype=torch.long)
    for i in range(len(lens)):
        tok[i, :lens[i]] = torch.from_numpy(ids[off[i]:off[i + 1]].astype(np.int64))
        att[i, :lens[i]] = 1
    with torch.no_grad():
        h = bert(input_ids=tok, attention_mask=att, token_type_ids=torch.zeros_like(tok)
                 ).last_hidden_state[:, 0].numpy()
    ref = h @ m.p["w_r"] + m.p["b_r"][0]
    assert np.max(np.abs(ours - ref)) <= 1e-10


def test_decoder_scores_match_gpt2_model():
    from transformers import GPT2Config, GPT2Model
    m = model(DEC)
    cfg = GPT2Config(vocab_size=DEC.vocab, n_positions=DEC.max_pos, n_embd=DEC.hidden,
                     n_layer=DEC.n_layers, n_head=DEC.n_heads, n_inner=DEC.ffn,
                     activation_function="gelu", resid_pdrop=0.0, embd_pdrop=0.0, attn_pdrop=0.0,
                     layer_norm_epsilon=DEC.ln_eps, attn_implementation="eager")
    gpt = GPT2Model(cfg).to(torch.float64).train(False)
    sd = {"wte.weight": m.p["emb_word"], "wpe.weight": m.p["emb_pos"],
          "ln_f.weight": m.p["lnf_g"], "ln_f.bias": m.p["lnf_b"]}
    for l, lw in enumerate(m.layers):
        p = f"h.{l}."
        sd[p + "ln_1.weight"] = lw["ln1_g"]
        sd[p + "ln_1.bias"] = lw["ln1_b"]
        sd[p + "attn.c_attn.weight"] = lw["w_qkv"].T      # Conv1D keeps [in][out]
        sd[p + "attn.c_attn.bias"] = lw["b_qkv"]
        sd[p + "attn.c_proj.weight"] = lw["w_o"].T
        sd[p + "attn.c_proj.bias"] = lw["b_o"]
        sd[p + "ln_2.weight"] = lw["ln2_g"]
        sd[p + "ln_2.bias"] = lw["ln2_b"]
        sd[p + "mlp.c_fc.weight"] = lw["w_1"].T
        sd[p + "mlp.c_fc.bias"] = lw["b_1"]
        sd[p + "mlp.c_proj.weight"] = lw["w_2"].T
        sd[p + "mlp.c_proj.bias"] = lw["b_2"]
    gpt.load_state_dict({k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in sd.items()},
                        strict=False)
    for L in (1, 5, 31):
        ids = ids_for(DEC, L, seed=L)
        ours = O.score_one(m, ids)
        with torch.no_grad():
            h = gpt(input_ids=torch.from_numpy(ids.astype(np.int64))[None]).last_hidden_state[0, -1]
        ref = float(h.numpy() @ m.p["w_r"] + m.p["b_r"][0])      # GPT2Model applies ln_f
        assert abs(ours - ref) <= 1e-10


# --- padding-free equals padded-and-masked --------------------------------------------

@pytest.mark.parametrize("shape", [ENC, DEC], ids=["enc", "dec"])
def test_packed_equals_padded(shape):
    m = model(shape)
    lens = np.array([3, 1, 17, 9, 30])
    off = synth.offsets_from_lengths(lens)
    ids = ids_for(shape, int(off[-1]), seed=4)
    a = O.score_packed(m, ids, off)
    b = O.score_padded(m, ids, off, pad_id=5)
    assert np.max(np.abs(a - b)) <= 1e-12


# --- closed forms and invariants ----------------------------------------------------

def test_attention_of_single_token_is_value_projection():
    m = model(ENC)
    lw = m.layers[0]
    H = ENC.hidden
    x = np.random.default_rng(8).normal(size=(1, H))
    v = x @ lw["w_qkv"][2 * H:].T + lw["b_qkv"][2 * H:]
    expect = v @ lw["w_o"].T + lw["b_o"]
    for causal in (False, True):
        assert np.max(np.abs(O.mha(x, lw, ENC.n_heads, causal) - expect)) <= 1e-13


@pytest.mark.parametrize("shape", [ENC, DEC], ids=["enc", "dec"])
def test_repeated_token_without_positions_scores_like_one_token(shape):
    m = model(shape)
    m.p["emb_pos"][:] = 0.0
    one = O.score_one(m, np.array([42]))
    for L in (2, 7, 33):
        assert abs(O.score_one(m, np.full(L, 42)) - one) <= 1e-12


def test_encoder_is_permutation_invariant_after_token0_without_positions():
    m = model(ENC)
    m.p["emb_pos"][:] = 0.0
    ids = ids_for(ENC, 12, seed=12)
    perm = np.concatenate([[0], 1 + np.random.default_rng(1).permutation(11)])
    assert abs(O.score_one(m, ids) - O.score_one(m, ids[perm])) <= 1e-12
    # but not when token 0 moves
    swapped = ids.copy()
    swapped[[0, 1]] = swapped[[1, 0]]
    assert abs(O.score_one(m, ids) - O.score_one(m, swapped)) > 1e-6


@pytest.mark.parametrize("shape", [ENC, DEC], ids=["enc", "dec"])
def test_head_relabelling_leaves_scores_unchanged(shape):
    m = model(shape)
    H, h = shape.hidden, shape.n_heads
    d = H // h
    ids = ids_for(shape, 15, seed=6)
    before = O.score_one(m, ids)
    perm = np.array([2, 0, 3, 1])
    cols = np.concatenate([np.arange(p * d, (p + 1) * d) for p in perm])
    for lw in m.layers:
        rows = np.concatenate([cols, H + cols, 2 * H + cols])
        lw["w_qkv"] = lw["w_qkv"][rows]
        lw["b_qkv"] = lw["b_qkv"][rows]
        lw["w_o"] = lw["w_o"][:, cols]
    assert abs(O.score_one(m, ids) - before) <= 1e-12


def test_decoder_is_causal():
    m = model(DEC)
    ids = ids_for(DEC, 20, seed=7)
    full = O.hidden_states(m, ids)
    for r in (0, 4, 13):
        part = O.hidden_states(m, ids[:r + 1])
        assert np.max(np.abs(full[:r + 1] - part)) <= 1e-12


@pytest.mark.parametrize("shape", [ENC, DEC], ids=["enc", "dec"])
def test_zero_gains_give_head_of_last_bias(shape):
    m = model(shape)
    last_b = m.layers[-1]["ln2_b"] if shape.arch == synth.ENC_POSTLN else m.p["lnf_b"]
    for lw in m.layers:
        lw["ln2_g"][:] = 0.0
    if shape.arch == synth.DEC_PRELN:
        m.p["lnf_g"][:] = 0.0
    expect = float(last_b @ m.p["w_r"] + m.p["b_r"][0])
    assert abs(O.score_one(m, ids_for(shape, 9)) - expect) <= 1e-13


def test_scores_are_sensitive_to_every_layer_term():
    """Dropping any one parameter tensor changes the score: no term is dead."""
    m = model(ENC)
    ids = ids_for(ENC, 11, seed=2)
    base = O.score_one(m, ids)
    for name in m.layers[0]:
        saved = m.layers[0][name].copy()
        m.layers[0][name] = m.layers[0][name] * 0.5
        assert abs(O.score_one(m, ids) - base) > 1e-6, name
        m.layers[0][name] = saved


def test_oracle_reproduces_stored_golden_scores():
    import os
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path.insert(0, os.path.join(here, "golden"))
    import make_golden
    gold = np.loadtxt(os.path.join(here, "golden", "tiny_enc_scores.txt"))
    assert np.max(np.abs(make_golden.tiny_enc_scores() - gold)) <= 1e-12
