"""The length-bucketed arena plan: buffers that are live together never share
bytes, and the peak stays within the reservation bound."""
import numpy as np
import pytest

import synth
import classifier_scoring_b200 as rm
from classifier_scoring_b200 import build
from tests.helpers import config_for


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def live_together(f1, l1, f2, l2):
    return f1 <= l2 and f2 <= l1


@pytest.mark.parametrize("shape", [synth.TINY, synth.BERT_BASE, synth.GPT_1P3B],
                         ids=["tiny", "bert", "gpt"])
def test_plans_never_overlap_live_buffers(shape):
    cfg = config_for(shape, max_len=min(512, shape.max_pos))
    rng = np.random.default_rng(0)
    for _ in range(200):
        T = int(rng.integers(1, 40000))
        S = int(rng.integers(0, 200_000_000))
        off, nb, first, last, peak = rm.ops.arena_plan(cfg, T, 1, S)
        for a in range(len(off)):
            assert off[a] % 256 == 0
            for b in range(a + 1, len(off)):
                if nb[a] and nb[b] and live_together(first[a], last[a], first[b], last[b]):
                    assert off[a] + nb[a] <= off[b] or off[b] + nb[b] <= off[a], (a, b, T, S)
        assert peak == max(int(o + n) for o, n in zip(off, nb))
        # never worse than no sharing, never better than the largest live set
        assert peak <= int(nb.sum())
        live = max(sum(int(nb[k]) for k in range(len(nb)) if first[k] <= s <= last[k])
                   for s in range(10))
        assert peak >= live


def test_sharing_saves_memory_on_bert():
    cfg = config_for(synth.BERT_BASE, max_len=100)
    T = 3264
    S = 12 * 64 * 51 * 56
    off, nb, first, last, peak = rm.ops.arena_plan(cfg, T, 64, S)
    assert peak < 0.75 * int(nb.sum())


def test_decoder_plans_no_sublayer_output_buffers():
    """The decoder adds its out-projection and FFN2 outputs straight into its
    fp32 residual stream, so its plans give y1 and y2 (buffers 5 and 7) no
    bytes; the encoder's keep one bf16 row per token each."""
    T, S = 3000, 0
    dec = config_for(synth.GPT_1P3B, max_len=560)
    off, nb, first, last, peak = rm.ops.arena_plan(dec, T, 8, S)
    assert nb[5] == 0 and nb[7] == 0
    assert nb[0] == T * synth.GPT_1P3B.hidden * 4          # x in fp32
    enc = config_for(synth.BERT_BASE, max_len=100)
    off, nb, first, last, peak = rm.ops.arena_plan(enc, T, 64, S)
    assert nb[5] == nb[7] == T * synth.BERT_BASE.hidden * 2
