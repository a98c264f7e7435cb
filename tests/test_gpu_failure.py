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
