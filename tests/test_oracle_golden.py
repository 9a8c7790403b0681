"""The oracle against its frozen results on three tiny seeded layers (bf16,
fp8, MXFP4 weights), written by tests/golden/make_golden.py. The pages print no
worked example; these fixtures are a tripwire: a change to the oracle's
arithmetic must regenerate them and say which reading of the pages justifies
it. CPU only."""
import json
import os
import sys

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_golden  # noqa: E402


@pytest.mark.parametrize("name", sorted(make_golden.CASES))
def test_oracle_matches_its_golden_fixture(name):
    with open(os.path.join(HERE, "golden", name + ".json")) as f:
        want = json.load(f)
    got = make_golden.compute(make_golden.CASES[name])
    assert got["config"] == want["config"]
    assert got["topk_ids"] == want["topk_ids"]
    assert got["topk_weights"] == want["topk_weights"]
    # outputs: bf16 values; a BLAS with another summation order may move one
    # across a rounding boundary, so one bf16 step (2^-7 relative) is allowed
    g = np.array([[float.fromhex(v) for v in row] for row in got["out"]])
    w = np.array([[float.fromhex(v) for v in row] for row in want["out"]])
    assert np.all(np.abs(g - w) <= np.abs(w) * 2.0**-7 + 1e-30)
    assert np.mean(g == w) > 0.99
