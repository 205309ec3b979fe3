"""The oracle still reproduces its frozen results on the tiny workload.

tests/golden/tiny_oracle.json was written by tests/golden/make_golden.py, which
calls only the oracle and the input generator.
"""
import json
import os

import pytest

from tests.golden import make_golden

pytestmark = pytest.mark.filterwarnings("ignore")


def test_oracle_matches_frozen_fixture():
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")) as f:
        frozen = json.load(f)
    assert make_golden.compute() == frozen
