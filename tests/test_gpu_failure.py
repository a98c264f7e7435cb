"""Failure detection without a GPU fault: a bounded wait that nothing ends
gives up at its limit, reports it, and the context keeps working."""
import numpy as np
import pytest
import torch

import classifier_scoring_b200 as rm
from oracle import scorer as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    limit = 50_000_000                                  # 50 ms
    timed_out, ns = rm.selftest_bounded_wait(limit)
    assert timed_out == 1
    assert limit <= ns < 20 * limit
    # the same context still runs the GEMM correctly
    g = torch.Generator().manual_seed(3)
    x = torch.randn(300, 256, generator=g).to(torch.bfloat16)
    w = (torch.randn(512, 256, generator=g) * 0.05).to(torch.bfloat16)
    y = torch.empty(300, 512, dtype=torch.float32, device="cuda")
    rm.ops.gemm(x.cuda(), w.cuda(), None, y, rm.F32, 300, 512, 256, 0)
    torch.cuda.synchronize()
    ref = O.linear(x.double().numpy(), w.double().numpy(), None)
    scale = np.abs(x.double().numpy()) @ np.abs(w.double().numpy()).T
    assert np.all(np.abs(y.double().cpu().numpy() - ref) <= 1e-5 * scale)


def test_selftest_rejects_bad_limits():
    with pytest.raises(rm.RmError):
        rm.selftest_bounded_wait(10)


def test_injected_allocation_failures_release_everything_and_leave_handles_usable():
    """Every allocation that rm_create (5), rm_create_shared (3) and
    rm_plan_create (1) make is failed in turn: each call returns RM_E_NOMEM,
    the device's free memory comes back to where it was (a leak of the
    weights, their staging or the arena would show: each is tens of MB here),
    and the next call without a failure succeeds and scores like the oracle."""
    import synth
    from tests.helpers import SCORE_ATOL, config_for, oracle_model

    shape = synth.TINYBERT
    flat = synth.make_weights(shape, 1)
    cfg = config_for(shape, max_batch_seqs=8, max_tokens=16384, max_len=256)
    lens = np.array([7, 64, 1, 130])
    off = synth.offsets_from_lengths(lens)
    ids = synth.make_token_ids(int(off[-1]), shape.vocab, 21)
    ids_d = torch.from_numpy(ids).cuda()

    def scores(sc):
        out = torch.full((len(lens),), float("nan"), device="cuda")
        sc.score(ids_d, off, out)
        torch.cuda.synchronize()
        return out.cpu().numpy().astype(np.float64)

    # one full cycle first: lazily loaded kernels and the context's local-memory
    # reservation stay with the context and must not count as a leak
    warm = rm.Scorer(cfg, flat)
    scores(warm)
    warm.shared().close()
    warm.plan(off).close()
    warm.close()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    try:
        for k in range(1, 6):
            rm.debug_fail_alloc(k)
            with pytest.raises(rm.RmError) as e:
                rm.Scorer(cfg, flat)
            assert e.value.code == rm.RM_E_NOMEM, (k, e.value)
            torch.cuda.synchronize()
            assert torch.cuda.mem_get_info()[0] >= free0 - (2 << 20), k
        rm.debug_fail_alloc(0)
        sc = rm.Scorer(cfg, flat)
        base = scores(sc)
        m = oracle_model(shape, flat)
        ref = np.array([O.score_one(m, ids[off[i]:off[i + 1]]) for i in range(len(lens))])
        assert np.max(np.abs(base - ref)) <= SCORE_ATOL
        for k in range(1, 4):
            rm.debug_fail_alloc(k)
            with pytest.raises(rm.RmError) as e:
                sc.shared()
            assert e.value.code == rm.RM_E_NOMEM, (k, e.value)
        rm.debug_fail_alloc(1)
        with pytest.raises(rm.RmError) as e:
            sc.plan(off)
        assert e.value.code == rm.RM_E_NOMEM
        rm.debug_fail_alloc(0)
        assert np.array_equal(scores(sc), base)          # the handle is untouched
        other = sc.shared()
        assert np.array_equal(scores(other), base)
        plan = sc.plan(off)
        out = torch.full((len(lens),), float("nan"), device="cuda")
        plan.score(ids_d, out)
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy().astype(np.float64), base)
        plan.close()
        other.close()
        sc.close()
    finally:
        rm.debug_fail_alloc(0)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free0 - (2 << 20)


def test_debug_fail_alloc_rejects_negative_counts():
    with pytest.raises(rm.RmError) as e:
        rm.debug_fail_alloc(-1)
    assert e.value.code == rm.RM_E_INVAL
