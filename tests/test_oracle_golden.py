"""Regression pins: the oracles still reproduce tests/golden/tiny_layer.json
and tiny_mlp.json (written by tests/golden/make_golden.py from the oracles
alone)."""
import json
import os

import numpy as np

from tests.golden.make_golden import compute

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_stored_tiny_case():
    with open(os.path.join(HERE, "golden", "tiny_layer.json")) as f:
        ref = json.load(f)
    now = compute()
    for key in ("y", "dx", "dA_q", "dB_o"):
        np.testing.assert_allclose(np.array(now[key]), np.array(ref[key]), rtol=1e-12, atol=1e-13)


def test_mlp_oracle_matches_stored_tiny_case():
    from tests.golden.make_golden import compute_mlp
    with open(os.path.join(HERE, "golden", "tiny_mlp.json")) as f:
        ref = json.load(f)
    now = compute_mlp()
    for key in ("y", "dx", "dA_up", "dB_down"):
        np.testing.assert_allclose(np.array(now[key]), np.array(ref[key]), rtol=1e-12, atol=1e-13)
