"""Regression check of the oracle against tests/golden/oracle_small.json."""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("name", ["linear", "ln", "mlp"])
def test_oracle_matches_golden(name):
    from tests.golden.make_golden import run_case
    ref = json.load(open(os.path.join(HERE, "golden", "oracle_small.json")))["outputs"][name]
    got = run_case(name)
    for k, v in ref.items():
        np.testing.assert_allclose(np.array(got[k]), np.array(v), rtol=1e-12, atol=1e-14)
