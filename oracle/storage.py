"""Storage rounding of the oracle.  Test infrastructure only.

The bf16 workloads store features, queries, keys and the coupled features h'
in bfloat16 (the workloads' own specification: "bf16 storage, fp32
accumulate"); the oracle computes in float64 and, where a stored value is
modelled, rounds its own float64 result with this function.  Pinned against
torch's float32 -> bfloat16 conversion, ties included
(tests/test_oracle_projection.py).
"""
from __future__ import annotations

import numpy as np


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Values rounded to bfloat16 (8 significant bits, round half to even) and
    returned as float64.  Exact for normal numbers in float32's exponent range
    (the only ones these inputs hold); no subnormal or overflow handling."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                    # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)
