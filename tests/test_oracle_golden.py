"""The oracle's stage outputs on the tiny workload match the committed fixture
written by tests/golden/make_golden.py (which calls only the oracle)."""
import json
import os

import pytest

from tests.golden import make_golden

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("key,m,balanced", [("f4_identity", 4, False), ("f6_rownorm", 6, True)])
def test_oracle_matches_golden_digests(key, m, balanced):
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        want = json.load(f)[key]
    got = make_golden.case(m, balanced)
    assert got == want
