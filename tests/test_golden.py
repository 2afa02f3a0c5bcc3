"""The oracle still reproduces the outputs frozen by tests/golden/make_golden.py."""
import json
import os
import sys

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
sys.path.insert(0, GOLDEN)


def test_oracle_matches_frozen_outputs():
    import make_golden
    want = json.load(open(os.path.join(GOLDEN, "oracle_regression.json")))
    got = make_golden.build()
    assert got["mask_tau1"] == want["mask_tau1"] and got["mask_q070"] == want["mask_q070"]
    assert got["e4m3_codes_linspace_-500_500_257"] == want["e4m3_codes_linspace_-500_500_257"]
    for t, vals in want["attention"].items():
        a = [float.fromhex(x) for x in got["attention"][t]]
        b = [float.fromhex(x) for x in vals]
        assert max(abs(x - y) for x, y in zip(a, b)) < 1e-12
    assert got["tau_q070"] == want["tau_q070"]
