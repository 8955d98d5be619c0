"""The oracle still reproduces its frozen tiny-workload digest (see
tests/golden/make_golden.py for how and why it was written)."""
import json
import os

import numpy as np

from tests.golden.make_golden import digest

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_frozen_digest():
    with open(os.path.join(HERE, "c0_oracle.json")) as f:
        ref = json.load(f)
    now = digest()
    for key, val in ref.items():
        if key == "workload":
            continue
        np.testing.assert_allclose(np.asarray(now[key]), np.asarray(val), rtol=1e-9, atol=1e-12,
                                   err_msg=key)
