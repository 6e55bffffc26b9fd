"""The oracle's stage outputs on the tiny workload match the committed fixture
written by tests/golden/make_golden.py (which calls only the oracle)."""
import json
import os

import pytest

from tests.golden import make_golden

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("key,m,balanced,opts", [
    ("f4_identity", 4, False, {}), ("f6_rownorm", 6, True, {}),
    ("f6_rownorm_y_tap", 6, True, {"per_tap": True}), ("f6_rownorm_x_int8", 6, True, {"x_int8": True}),
    ("f6_rownorm_int8_transforms", 6, True, {"int8_transforms": True}),
])
def test_oracle_matches_golden_digests(key, m, balanced, opts):
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        want = json.load(f)[key]
    got = make_golden.case(m, balanced, **opts)
    assert got == want
