"""Edge-centric eSCN convolution of the oracle.  Test infrastructure only.

"EquiformerV3: Scaling Efficient, Expressive, and General SE(3)-Equivariant
Graph Attention Transformers", section "eSCN卷积与SO(2)线性层": eSCN splits a tensor product into two steps — rotate the features by
D_ij, the rotation that the relative position r_ij defines, then apply an
SO(2) linear layer that acts only within the 2l+1 components of each degree
(with components of order |m| > M_max dropped).  It is the edge-centric
formulation that the on-the-fly attention's node-centric factorisation
replaces ("E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §1, §3.2).

Readings taken where the page is silent (the plainest ones):

* r_ij = r_j - r_i, Q_ij the alignment rotation of r_ij (Q_ij z^ = r^_ij,
  ZYZ with zero roll, identity for r_ij = 0), x~ = D(Q_ij)^T h_j into the
  edge frame and D(Q_ij) y~ back out — the EAAS convention of this project;
* the SO(2) linear layer acts per feature channel c (no channel mixing), on
  each order m separately, mixing degrees:
      y~^lo_0  = sum_li W0[lo][li][c] x~^li_0
      y~^lo_+m = sum_li (W1_m[lo][li][c] x~^li_+m - W2_m[lo][li][c] x~^li_-m)
      y~^lo_-m = sum_li (W2_m[lo][li][c] x~^li_+m + W1_m[lo][li][c] x~^li_-m)
  for 1 <= m <= min(M_max, lo, li); orders above M_max are zero.  The 2x2
  blocks [[W1, -W2], [W2, W1]] commute with rotations about the edge axis,
  which is what makes the layer SO(2)- and the whole message SO(3)-equivariant;
* the weights are fixed inputs (eSCN's radial networks, which make them
  depend on |r_ij|, belong to the model around the operation);
* messages are summed over the neighbour list: out_i = sum_j D(Q_ij) y~_ij.

Weight layout float32 [NW][C]: W0 [(L+1)^2] at row lo*(L+1) + li, then for
m = 1..M_max the (L+1-m)^2 entries of W1_m followed by those of W2_m, each at
row (lo-m)*(L+1-m) + (li-m) of its block.

Pins (tests/test_oracle_escn.py): identity weights give the neighbour sum of
h; a degree-1 m = 0 projector gives sum_j (r^_ij . h_j) r^_ij; the result does
not depend on the roll angle of Q_ij; global rotation equivariance.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from . import so3


def num_weights(L: int, mmax: int) -> int:
    return (L + 1) ** 2 + sum(2 * (L + 1 - m) ** 2 for m in range(1, mmax + 1))


def weight_rows(L: int, mmax: int):
    """(W0, [(W1_m, W2_m) for m = 1..mmax]) as row-index arrays into [NW][C]."""
    w0 = np.arange((L + 1) ** 2).reshape(L + 1, L + 1)
    off = (L + 1) ** 2
    blocks = []
    for m in range(1, mmax + 1):
        n = L + 1 - m
        w1 = off + np.arange(n * n).reshape(n, n)
        w2 = off + n * n + np.arange(n * n).reshape(n, n)
        blocks.append((w1, w2))
        off += 2 * n * n
    return w0, blocks


def so2_linear(xt: np.ndarray, w: np.ndarray, L: int, mmax: int) -> np.ndarray:
    """The SO(2) linear layer in the edge frame: xt [D, C] -> [D, C]."""
    w0, blocks = weight_rows(L, mmax)
    comp = lambda l, m: l * l + l + m
    y = np.zeros_like(xt)
    for lo in range(L + 1):
        for li in range(L + 1):
            y[comp(lo, 0)] += w[w0[lo, li]] * xt[comp(li, 0)]
            for m in range(1, min(mmax, lo, li) + 1):
                w1 = w[blocks[m - 1][0][lo - m, li - m]]
                w2 = w[blocks[m - 1][1][lo - m, li - m]]
                xp, xm = xt[comp(li, m)], xt[comp(li, -m)]
                y[comp(lo, m)] += w1 * xp - w2 * xm
                y[comp(lo, -m)] += w2 * xp + w1 * xm
    return y


def rotate_blocks(x: np.ndarray, Ds: Sequence[np.ndarray], transpose: bool) -> np.ndarray:
    """x [D, C] with each degree block multiplied by D^l (or its transpose)."""
    y = np.empty_like(x)
    for l, D in enumerate(Ds):
        blk = slice(l * l, (l + 1) * (l + 1))
        y[blk] = (D.T if transpose else D) @ x[blk]
    return y


def escn_conv(h, pos, w, L: int, mmax: int, nbrs: Sequence[np.ndarray],
              targets: Optional[Sequence[int]] = None, roll=None) -> np.ndarray:
    """out_i = sum_{j in N(i)} D(Q_ij) SO2(D(Q_ij)^T h_j) for each target i.

    h [N, D, C]; pos [N, 3]; w [NW, C]; nbrs[t] lists the neighbours of
    targets[t] (default: target t = atom t).  roll(i, j), if given, returns an
    angle gamma and Q_ij R_z(gamma) is used instead of Q_ij (a test of the
    layer's independence of the roll).  Returns [len(nbrs), D, C] float64.
    """
    h = np.asarray(h, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    N, D, C = h.shape
    assert D == (L + 1) ** 2 and w.shape == (num_weights(L, mmax), C)
    targets = list(range(len(nbrs))) if targets is None else list(targets)
    out = np.zeros((len(nbrs), D, C))
    for t, (i, js) in enumerate(zip(targets, nbrs)):
        for j in np.asarray(js, dtype=np.int64):
            Q = so3.alignment_rotation(pos[j] - pos[i])
            if roll is not None:
                Q = Q @ so3.rot_z(roll(i, j))
            Ds = [so3.wigner_D(l, Q) for l in range(L + 1)]
            xt = rotate_blocks(h[j], Ds, transpose=True)
            out[t] += rotate_blocks(so2_linear(xt, w, L, mmax), Ds, transpose=False)
    return out
