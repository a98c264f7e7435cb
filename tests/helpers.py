"""Shared helpers of the tests: configs from synthetic shapes, tolerances."""
import numpy as np

import synth
from classifier_scoring_b200 import RmConfig

# Final-score tolerance (absolute) and kernel-level fp32 tolerance (relative).
SCORE_ATOL = 2e-2
F32_RTOL = 1e-5


def config_for(shape: synth.ModelShape, *, max_batch_seqs=64, max_tokens=8192, max_len=None,
               sched_max_batch=64, sched_c0=0, sched_c1=1, sched_table=None,
               attn_impl=0, sched_objective=0, sched_max_cost=0) -> RmConfig:
    if max_len is None:
        max_len = min(shape.max_pos, 1024)
    return RmConfig.make(arch=shape.arch, n_layers=shape.n_layers, hidden=shape.hidden,
                         n_heads=shape.n_heads, ffn=shape.ffn, vocab=shape.vocab,
                         max_pos=shape.max_pos, weight_dtype=shape.weight_dtype, gelu=shape.gelu,
                         ln_eps=shape.ln_eps, max_batch_seqs=max_batch_seqs, max_tokens=max_tokens,
                         max_len=max_len, sched_max_batch=sched_max_batch, sched_c0=sched_c0,
                         sched_c1=sched_c1, sched_table=sched_table, attn_impl=attn_impl,
                         sched_objective=sched_objective, sched_max_cost=sched_max_cost)


def oracle_model(shape: synth.ModelShape, flat):
    from oracle import scorer
    return scorer.unpack_weights(flat, shape.arch, shape.n_layers, shape.hidden, shape.n_heads,
                                 shape.ffn, shape.vocab, shape.max_pos, shape.weight_dtype,
                                 shape.gelu, shape.ln_eps)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to the nearest bf16 (returned as float64)."""
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))).astype(np.float64)
