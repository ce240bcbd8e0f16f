"""The oracle's output on the tiny fp32 workload is frozen in tests/golden/tiny_fp32.json
(written by tests/golden/make_golden.py, which calls only the oracle and the input generator)."""
import json
import os

import numpy as np
import pytest

from tests.golden.make_golden import summarise

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_fp32.json")


@pytest.mark.slow
def test_oracle_matches_frozen_fixture():
    ref = json.load(open(GOLDEN))
    cur = summarise()
    assert cur["sel"] == ref["sel"]
    np.testing.assert_allclose(cur["M"], ref["M"], rtol=1e-10, atol=0)
    np.testing.assert_allclose(cur["o_sum"], ref["o_sum"], rtol=1e-10)
    np.testing.assert_allclose(cur["o_sumsq"], ref["o_sumsq"], rtol=1e-10)
    for a, b in zip(cur["o_samples"], ref["o_samples"]):
        assert a[:3] == b[:3]
        np.testing.assert_allclose(a[3], b[3], rtol=1e-10)
    np.testing.assert_allclose(cur["Hbar_trace"], ref["Hbar_trace"], rtol=1e-10)
