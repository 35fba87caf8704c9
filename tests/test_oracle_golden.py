"""The oracle's speedup model against the numbers the pages print.

tests/golden/pages_tpf.json holds each printed value with its source and the
rounding the page applies. The oracle's TPF formula (whose equality with the
block layout's renewal process is pinned in test_oracle_isd.py) must land on
every printed value, and TPF^2 / (2N - 1) on every printed efficiency, which
also pins the reading that a forward carries 2N - 1 queries.
"""
import json
import os

import pytest

from oracle import isd as oi

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_tpf.json")
with open(GOLDEN) as f:
    CASES = json.load(f)["cases"]


@pytest.mark.parametrize("case", CASES, ids=[f"{c['quantity']}-N{c['N']}-p{c['p']}-{i}"
                                             for i, c in enumerate(CASES)])
def test_printed_speedup_numbers(case):
    tpf = oi.tpf_formula(case["p"], case["N"])
    value = tpf if case["quantity"] == "tpf" else tpf ** 2 / (2 * case["N"] - 1)
    assert abs(value - case["printed"]) <= case["tol"], (value, case["cite"])
