"""The checked build (librmscore_checked.so: kernels bounds-check the indices
they derive from per-call metadata, count failures, skip the access).  Run in
child processes, since a process loads one build of the library."""
import json
import os
import subprocess
import sys

import pytest
import torch

import classifier_scoring_b200 as rm
from classifier_scoring_b200 import build as rmbuild
from tests.helpers import SCORE_ATOL

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def checked_lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return rmbuild.build(checked=True)


def run_case(case):
    env = dict(os.environ, RMSCORE_LIB=rm.CHECKED_LIB_PATH, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "tests.checked_cases", case], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_checked_build_scores_like_the_oracle_with_no_failed_bound():
    """Config-1 shapes (the tiny encoder) and a small decoder through every
    attention path: scores within the tolerance, no failed bounds test."""
    res = run_case("valid")
    assert res["checked"] == 1
    assert res["bounds_before"] == 0 and res["bounds_after"] == 0
    for k, v in res.items():
        if k.endswith(("_err_0", "_err_1")):
            assert v <= SCORE_ATOL, (k, v)


def test_checked_build_counts_inconsistent_metadata_and_stays_usable():
    res = run_case("invalid")
    assert res["bounds_before"] == 0
    assert res["head_bounds"] >= 1
    assert res["head_out"][1] != res["head_out"][1]          # the empty sequence's slot untouched (NaN)
    assert res["head_out"][0] == res["head_out"][0] and res["head_out"][2] == res["head_out"][2]
    assert res["softmax_bounds"] >= 1
    assert res["tiny_err_0"] <= SCORE_ATOL and res["tiny_err_1"] <= SCORE_ATOL


def test_product_build_reports_no_checks():
    assert not rm.build_checked()
    assert rm.bounds_errors() == 0
