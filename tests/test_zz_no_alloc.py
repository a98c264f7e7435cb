"""rm_op_attention_noalloc: the attention step for callers that cannot
allocate device memory where they run it (a plugin inside a runtime that owns
the memory pool, or a path where cudaMalloc may not be called).  Its scratch
is a fixed array inside the library, so this file checks it against the
existing caller-allocated entry points (the same kernels: the results must be
bit-identical) on two calls in a row, against the fp64 oracle, at the edges of
its documented limits, and one past each limit.  Kept last in collection order
so that a run stopping at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import synth
import classifier_scoring_b200 as rm
from oracle import scorer as O

pytestmark = pytest.mark.gpu
BF16_REL = 2.0 ** -8
F32_RTOL = 1e-5


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


def noalloc_ctx(qkv, off, nh, d, causal):
    T = int(off[-1])
    out = torch.full((T, nh * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    rm.ops.attention_noalloc(qkv, out, off, nh, d, causal)
    torch.cuda.synchronize()
    return out


def check_against_oracle(qkv, ctx, off, nh, d, causal):
    """fp64 attention of the oracle on the same bf16 q, k, v.  The path stores
    the scores s and the probabilities p in bf16 (half an ulp, 2^-9 relative,
    each) and rounds the output once: a score error of 2^-9 |s| moves p_c by
    at most p_c * 2^-8 * max|s| (the softmax's own shift included), so per
    output the bound is 2^-8 |ref| + (2^-8 max|s| + 2^-8) (p @ |v|) plus the
    fp32 accumulation (1e-5 relative)."""
    X = qkv.double().cpu().numpy()
    C = ctx.double().cpu().numpy()
    H = nh * d
    for i in range(len(off) - 1):
        rows = X[off[i]:off[i + 1]]
        for j in range(nh):
            q = rows[:, j * d:(j + 1) * d]
            k = rows[:, H + j * d:H + (j + 1) * d]
            v = rows[:, 2 * H + j * d:2 * H + (j + 1) * d]
            p = O.attention_probs(q, k, bool(causal))
            ref = p @ v
            smax = float(np.max(np.abs(q @ k.T))) / np.sqrt(d)
            tol = BF16_REL * np.abs(ref) + (BF16_REL * smax + BF16_REL) * (p @ np.abs(v)) + F32_RTOL
            got = C[off[i]:off[i + 1], j * d:(j + 1) * d]
            assert np.all(np.abs(got - ref) <= tol), (i, j, float((np.abs(got - ref) / tol).max()))


@pytest.mark.parametrize("causal", [0, 1])
def test_two_calls_in_a_row_match_the_caller_allocated_path(causal):
    nh, d = 12, 64
    H = nh * d
    rng = np.random.default_rng(11 + causal)
    for call, lens in enumerate(([37, 1, 100, 64, 65, 2], [129, 7, 300, 50])):
        off = synth.offsets_from_lengths(np.array(lens))
        T = int(off[-1])
        qkv = torch.from_numpy(rng.normal(0, 1.5, (T, 3 * H))).to(torch.bfloat16).cuda()
        want = reference_ctx(qkv, off, nh, d, causal)
        got = noalloc_ctx(qkv, off, nh, d, causal)
        assert torch.equal(got, want), call
        check_against_oracle(qkv, got, off, nh, d, causal)


def test_exactly_the_score_limit():
    """One 512-token sequence with 16 heads fills the 4 Mi score entries exactly."""
    nh, d, L = 16, 64, 512
    assert nh * L * L == 4 * 1024 * 1024
    off = synth.offsets_from_lengths(np.array([L]))
    rng = np.random.default_rng(5)
    qkv = torch.from_numpy(rng.normal(0, 1.0, (L, 3 * nh * d))).to(torch.bfloat16).cuda()
    got = noalloc_ctx(qkv, off, nh, d, 0)
    assert torch.equal(got, reference_ctx(qkv, off, nh, d, 0))
    check_against_oracle(qkv, got, off, nh, d, 0)
    # one more token (16 heads * 1 * 8 padded entries) is past the limit
    with pytest.raises(rm.RmError) as e:
        rm.ops.attention_noalloc(qkv, got, synth.offsets_from_lengths(np.array([L, 1])), nh, d, 0)
    assert e.value.code == rm.RM_E_RANGE


def test_the_maximum_number_of_sequences():
    """4096 one-token sequences (the metadata's capacity), then 4097."""
    nh, d, n = 12, 64, 4096
    off = synth.offsets_from_lengths(np.ones(n, dtype=np.int64))
    rng = np.random.default_rng(6)
    qkv = torch.from_numpy(rng.normal(0, 1.0, (n, 3 * nh * d))).to(torch.bfloat16).cuda()
    got = noalloc_ctx(qkv, off, nh, d, 1)
    assert torch.equal(got, reference_ctx(qkv, off, nh, d, 1))
    # a one-token sequence attends to itself alone: the output is its own v, rounded once
    v = qkv[:, 2 * nh * d:]
    assert torch.equal(got, v)
    with pytest.raises(rm.RmError) as e:
        rm.ops.attention_noalloc(qkv, got, synth.offsets_from_lengths(np.ones(n + 1, dtype=np.int64)),
                                 nh, d, 1)
    assert e.value.code == rm.RM_E_RANGE


def test_calls_beyond_the_scratch_limit_are_rejected():
    nh, d = 16, 64
    off = synth.offsets_from_lengths(np.array([1024] * 300))      # 16 * 300 * 1024^2 entries
    qkv = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RmError) as e:
        rm.ops.attention_noalloc(qkv, qkv, off, nh, d, 0)
    assert e.value.code == rm.RM_E_RANGE
    assert "scratch" in str(e.value)
