"""The oracle still reproduces its stored outputs for the tiny fp32 workload."""
import json
import os

import numpy as np

from tests.golden import make_golden

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_stored_golden():
    stored = json.load(open(os.path.join(HERE, "config1_oracle.json")))
    now = make_golden.compute()
    assert now["shape"] == stored["shape"]
    np.testing.assert_allclose(now["out_row0_head0"], stored["out_row0_head0"], rtol=1e-12)
    np.testing.assert_allclose(now["out_row7_head1"], stored["out_row7_head1"], rtol=1e-12)
    np.testing.assert_allclose(now["out_sum"], stored["out_sum"], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(now["out_abs_sum"], stored["out_abs_sum"], rtol=1e-12)
