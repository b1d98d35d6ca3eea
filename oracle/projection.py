"""Invariant query/key projection of the oracle.  Test infrastructure only.

"E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation Memory"
§2.2 (node-centric factorisation, Eq. 6): queries and keys are SO(3)-invariant
scalar projections of the node features, and equivariant geometry travels
only along the value path.  The page names the projection but prints no
formula.  Reading taken (the plainest one): the invariant scalars of an atom
are its degree-0 channels h_i^(0) (C values, a rotation leaves them
unchanged), and each is mapped linearly, without bias, to every head:

    q_i[h][d] = sum_c h_i^(0)[c] wq[c][h*dk + d]
    k_i[h][d] = sum_c h_i^(0)[c] wk[c][h*dk + d]

with wq, wk float32 [C][H*dk].  Logits q_i . k_j / sqrt(dk) are then invariant
scalars, as the page requires.  Features [N, (lmax+1)^2, C] with component
l^2 + l + m; the degree-0 block is component 0.

Pins (tests/test_oracle_projection.py): a one-hot weight picks one input
channel into one (head, component) slot; a pure-Python triple loop on tiny
inputs; invariance of q, k and the logits when every degree block of h is
rotated by its Wigner-D matrix; the composed forward with projected q, k is
rotation-equivariant.
"""
from __future__ import annotations

import numpy as np

from .storage import round_bf16  # noqa: F401  (q and k storage of the bf16 workloads)


def invariant_projection(h: np.ndarray, wq: np.ndarray, wk: np.ndarray, H: int, dk: int):
    """(q, k), each [N, H, dk] float64, from the degree-0 channels of h."""
    h = np.asarray(h, dtype=np.float64)
    wq = np.asarray(wq, dtype=np.float64)
    wk = np.asarray(wk, dtype=np.float64)
    N, _, C = h.shape
    assert wq.shape == (C, H * dk) and wk.shape == (C, H * dk)
    h0 = h[:, 0, :]                       # invariant scalars [N, C]
    return (h0 @ wq).reshape(N, H, dk), (h0 @ wk).reshape(N, H, dk)
