"""The oracle still reproduces its stored regression set (CPU only)."""
import json
import os

import pytest

from tests.golden.make_regression import CASES, run_case

HERE = os.path.dirname(os.path.abspath(__file__))
STORED = json.load(open(os.path.join(HERE, "golden", "oracle_regression.json")))["cases"]


@pytest.mark.parametrize("name,over", CASES, ids=[c[0] for c in CASES])
def test_oracle_regression(name, over):
    got = run_case(name, over)
    ref = STORED[name]
    assert got["config"] == ref["config"]
    assert got["ids"] == ref["ids"]
    assert got["out_sum"] == pytest.approx(ref["out_sum"], rel=1e-12, abs=1e-12)
    assert got["out_abs_sum"] == pytest.approx(ref["out_abs_sum"], rel=1e-12)
    assert got["out_first_row"] == pytest.approx(ref["out_first_row"], rel=1e-12, abs=1e-12)
