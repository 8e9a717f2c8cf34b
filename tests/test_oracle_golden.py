"""The oracle still reproduces its committed regression fixture on the tiny workload."""
import json
import os

import numpy as np

from tests.golden import make_golden

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_tiny_step.json")


def test_oracle_tiny_step_regression():
    want = json.load(open(HERE))
    got = make_golden.compute()
    assert got["hidden_shape"] == want["hidden_shape"]
    np.testing.assert_allclose(got["hidden_sum"], want["hidden_sum"], rtol=1e-10, atol=1e-9)
    np.testing.assert_allclose(got["hidden_sumsq"], want["hidden_sumsq"], rtol=1e-10)
    for g, w in zip(got["samples"], want["samples"]):
        assert g["index"] == w["index"]
        np.testing.assert_allclose(g["value"], w["value"], rtol=1e-10, atol=1e-12)
