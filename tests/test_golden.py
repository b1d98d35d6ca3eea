"""Golden fixtures (CPU only).

* ``cg_textbook_1x1.txt``: the standard printed table of Clebsch–Gordan
  coefficients for two l = 1 states, against the oracle's Racah formula.
* ``forward_tiny.json``, ``backward_tiny.json``: the oracle's own output and
  gradients for a tiny seeded system, written by ``make_golden.py``;
  regression locks on the oracle.
"""
import json
import os
from fractions import Fraction

import numpy as np

from oracle import so3
from tests.golden.make_golden import build, build_backward

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_cg_textbook_table():
    seen = set()
    with open(os.path.join(HERE, "cg_textbook_1x1.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            m1, m2, J, M, v = line.split()
            m1, m2, J, M = int(m1), int(m2), int(J), int(M)
            sign = -1.0 if v.startswith("-") else 1.0
            val = sign * np.sqrt(float(Fraction(v.lstrip("+-"))))
            assert abs(so3.cg_complex(1, m1, 1, m2, J, M) - val) < 1e-15
            seen.add((m1, m2, J, M))
    for m1 in (-1, 0, 1):
        for m2 in (-1, 0, 1):
            for J in (0, 1, 2):
                if (m1, m2, J, m1 + m2) not in seen:
                    assert so3.cg_complex(1, m1, 1, m2, J, m1 + m2) == 0.0


def test_forward_tiny_regression():
    with open(os.path.join(HERE, "forward_tiny.json")) as f:
        rec = json.load(f)
    wl, d, nbrs, full, out = build()
    assert [n.tolist() for n in nbrs] == rec["neighbours"]
    assert full.tolist() == rec["full_degree"]
    assert np.max(np.abs(out - np.array(rec["out"]))) < 1e-12 * np.max(np.abs(out))


def test_backward_tiny_regression():
    with open(os.path.join(HERE, "backward_tiny.json")) as f:
        rec = json.load(f)
    _, dh, dq, dk, dr = build_backward()
    for name, got in (("dh", dh), ("dq", dq), ("dk", dk), ("dr", dr)):
        ref = np.array(rec[name])
        assert ref.shape == got.shape
        assert np.max(np.abs(got - ref)) < 1e-12 * max(1.0, np.max(np.abs(ref))), name
