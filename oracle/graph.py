"""Brute-force radius graph of the oracle.  Test infrastructure only.

[EX] §5.1 sets edge_cutoff 5.0 Å and §5.2 asks that the neighbour list be
verified.  The plainest exact reading: atom j is a neighbour of i when j != i
and |p_j - p_i|^2 <= r_c^2, evaluated in exact integer arithmetic on grid
coordinates.  A padded list of K slots keeps the K nearest, ties broken by
the smaller index.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np


def neighbours_of(pos_q: np.ndarray, cutoff_q: int, i: int) -> np.ndarray:
    """All neighbours of atom i ordered by (squared distance, index)."""
    P = np.asarray(pos_q, dtype=np.int64)
    d = P - P[i]
    d2 = np.sum(d * d, axis=1)
    rc2 = int(cutoff_q) * int(cutoff_q)
    js = np.nonzero(d2 <= rc2)[0]
    js = js[js != i]
    order = np.lexsort((js, d2[js]))
    return js[order]


def radius_graph(pos_q: np.ndarray, cutoff_q: int, K: Optional[int] = None,
                 rows: Optional[Sequence[int]] = None) -> Tuple[List[np.ndarray], np.ndarray]:
    """Neighbour lists for ``rows`` (default: all atoms).

    Returns (lists, full_degree): lists[t] holds the kept neighbours of row t
    ordered by (squared distance, index), truncated to K when K is given;
    full_degree[t] is the untruncated neighbour count.
    """
    n = np.asarray(pos_q).shape[0]
    rows = range(n) if rows is None else rows
    lists, full = [], []
    for i in rows:
        js = neighbours_of(pos_q, cutoff_q, int(i))
        full.append(len(js))
        lists.append(js if K is None else js[:K])
    return lists, np.asarray(full, dtype=np.int64)
