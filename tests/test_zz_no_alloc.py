"""rm_op_attention_noalloc: the attention step for callers that cannot
allocate device memory where they run it (a plugin inside a runtime that owns
the memory pool, or a path where cudaMalloc may not be called).  Its scratch
is a fixed array inside the library, so this file checks it against the
existing caller-allocated entry points on two calls in a row, and checks the
size limit.  Kept last in collection order so that a run stopping at the
first failure has already run every other test."""
import numpy as np
import pytest
import torch

import synth
import classifier_scoring_b200 as rm

pytestmark = pytest.mark.gpu
BF16_REL = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def reference_ctx(qkv, off, nh, d, causal):
    """The same step through rm_op_attn_scores / rm_op_softmax / rm_op_attn_context
    with a caller-allocated score buffer."""
    rb, so = rm.ops.varlen_meta(off, nh)
    S = torch.empty(int(so[-1]), dtype=torch.bfloat16, device="cuda")
    d_off = torch.from_numpy(off).cuda()
    d_rb = torch.from_numpy(rb).cuda()
    d_so = torch.from_numpy(so).cuda()
    T = int(off[-1])
    ctx = torch.zeros(T, nh * d, dtype=torch.bfloat16, device="cuda")
    n = len(off) - 1
    rm.ops.attn_scores(qkv, S, d_off, d_rb, d_so, n, int(rb[-1]), nh, d, causal)
    rm.ops.softmax(S, rm.BF16, d_off, d_so, n, T, nh, int(np.diff(off).max()), causal)
    rm.ops.attn_context(S, qkv, ctx, d_off, d_rb, d_so, n, int(rb[-1]), nh, d, causal)
    torch.cuda.synchronize()
    return ctx


@pytest.mark.parametrize("causal", [0, 1])
def test_two_calls_in_a_row_match_the_caller_allocated_path(causal):
    nh, d = 12, 64
    H = nh * d
    rng = np.random.default_rng(11 + causal)
    for call, lens in enumerate(([37, 1, 100, 64, 65, 2], [129, 7, 300, 50])):
        off = synth.offsets_from_lengths(np.array(lens))
        T = int(off[-1])
        qkv = torch.from_numpy(rng.normal(0, 1.5, (T, 3 * H))).to(torch.bfloat16).cuda()
        want = reference_ctx(qkv, off, nh, d, causal).double().cpu().numpy()
        got_t = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        rm.ops.attention_noalloc(qkv, got_t, off, nh, d, causal)
        torch.cuda.synchronize()
        got = got_t.double().cpu().numpy()
        assert np.all(np.isfinite(got)), call
        assert np.all(np.abs(got - want) <= BF16_REL * np.abs(want) + 1e-6), call


def test_calls_beyond_the_scratch_limit_are_rejected():
    nh, d = 16, 64
    off = synth.offsets_from_lengths(np.array([1024] * 300))      # 16 * 300 * 1024^2 entries
    qkv = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RmError) as e:
        rm.ops.attention_noalloc(qkv, qkv, off, nh, d, 0)
    assert e.value.code == rm.RM_E_RANGE
    assert "scratch" in str(e.value)
