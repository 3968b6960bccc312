"""The tiny Complex-KDA golden fixture (written by tests/golden/make_golden.py
from the oracle) still matches both the input generator and the oracle."""
import os
import sys

import numpy as np

import oracle
from workloads import tiny_ckda

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))
from make_golden import input_digest  # noqa: E402

GOLDEN = os.path.join(HERE, "golden", "tiny_ckda_seed0.txt")


def _parse():
    vals, o_rows, s_rows = {}, {}, {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split()
        if parts[0] == "o":
            t, h = int(parts[1][2:]), int(parts[2][2:])
            o_rows[(t, h)] = np.array([float(x) for x in parts[3:]])
        elif parts[0] == "S":
            h, i = int(parts[1][2:]), int(parts[2][4:])
            s_rows[(h, i)] = np.array([float(x) for x in parts[3:]])
        else:
            vals[parts[0]] = parts[1]
    return vals, o_rows, s_rows


def test_golden_tiny_ckda():
    vals, o_rows, s_rows = _parse()
    inp = tiny_ckda(0)
    assert input_digest(inp) == vals["inputs_sha256"]
    o, sf = oracle.recurrence(inp)
    assert abs(float(o.sum()) - float(vals["o_sum"])) < 1e-10
    assert abs(float((o ** 2).sum()) - float(vals["o_sq_sum"])) < 1e-9
    for (t, h), row in o_rows.items():
        np.testing.assert_allclose(o[0, t, h], row, rtol=0, atol=1e-13)
    for (h, i), row in s_rows.items():
        np.testing.assert_allclose(sf[0, h, i], row, rtol=0, atol=1e-13)
