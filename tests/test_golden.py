"""Regression pin: the oracle still reproduces the stored tiny-workload values."""

import json
import os

import numpy as np

from tests.golden.make_golden import build

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_oracle_fixture_reproduces():
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        stored = json.load(f)
    fresh = build()
    assert stored["workload"] == fresh["workload"]
    for a, b in zip(stored["probes"], fresh["probes"]):
        for key in ("q_prime", "k_prime", "o", "lse"):
            assert np.isclose(a[key], b[key], rtol=0, atol=1e-12), (a, key)
        assert a["q_code"] == b["q_code"]
    assert np.allclose(stored["q_scales"], fresh["q_scales"], rtol=0, atol=0)
    assert np.isclose(stored["o_sum"], fresh["o_sum"], rtol=1e-12)
    assert np.isclose(stored["o_sq_sum"], fresh["o_sq_sum"], rtol=1e-12)
