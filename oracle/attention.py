"""Dense coupling and two-pass attention of the oracle.  Test infrastructure only.

Follows the node-centric factorisation of [EX] §3.1:

1. source pre-coupling   h'_j = h_j (x) R(r_j)
2. streaming aggregation m_i  = sum_j alpha_ij h'_j
3. target coupling       ^h_i = m_i (x) R(r_i)

with the tensor product written out as the plain dense Clebsch–Gordan sum
([TS] §2.1 names it as the dense contraction that EAAS replaces), invariant
per-head logits q_i . k_j / sqrt(d_k) ([TS] §2.2, Eq. 6 makes q and k
invariant scalars), and a two-pass softmax over each atom's neighbours.

Readings where the pages are silent:

* the coupling weight w[p][c] multiplies path p of channel c; paths are all
  triangle-valid (li, lf, lo) up to lmax, odd li+lf+lo included;
* channel c belongs to head floor(c*H/C), the same for every degree;
* an atom without neighbours aggregates to m_i = 0;
* r_j is the atom's position vector as given (the inputs are centred on the
  system centroid).

Layouts: features [N, (lmax+1)^2, C] with component l^2+l+m; q, k [N, H, d_k];
weights [P, C] in ``so3.paths`` order.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from . import so3


def _block(x: np.ndarray, l: int) -> np.ndarray:
    return x[:, l * l:(l + 1) * (l + 1), :]


def tensor_product(x: np.ndarray, pos: np.ndarray, w: np.ndarray, lmax: int) -> np.ndarray:
    """y^{lo}[m][c] = sum_{p=(li,lf,lo)} w[p][c] sum_{mi,mf} T_p[m,mi,mf] x^{li}[mi][c] R^{lf}_{mf}(r).

    x [N, D, C]; pos [N, 3]; w [P, C].  Returns [N, D, C] float64.
    """
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    plist = so3.paths(lmax)
    assert w.shape[0] == len(plist)
    R = [so3.solid_harmonics(l, pos) for l in range(lmax + 1)]     # [N, 2l+1]
    y = np.zeros_like(x)
    for p, (li, lf, lo) in enumerate(plist):
        T = so3.real_cg(li, lf, lo)
        contrib = np.einsum("oif,nic,nf->noc", T, _block(x, li), R[lf])
        y[:, lo * lo:(lo + 1) * (lo + 1), :] += contrib * w[p][None, None, :]
    return y


def source_coupling(h, pos, w1, lmax):
    """h'_j = h_j (x) R(r_j) with weights w1 ([EX] §3.1 step 1)."""
    return tensor_product(h, pos, w1, lmax)


def target_coupling(m, pos, w2, lmax):
    """^h_i = m_i (x) R(r_i) with weights w2 ([EX] §3.1 step 3)."""
    return tensor_product(m, pos, w2, lmax)


def logits(q_i: np.ndarray, k_js: np.ndarray) -> np.ndarray:
    """s[j, h] = q_i[h] . k_j[h] / sqrt(d_k); q_i [H, dk], k_js [J, H, dk]."""
    q_i = np.asarray(q_i, dtype=np.float64)
    k_js = np.asarray(k_js, dtype=np.float64)
    return np.einsum("hd,jhd->jh", q_i, k_js) / np.sqrt(q_i.shape[-1])


def softmax_two_pass(s: np.ndarray) -> np.ndarray:
    """alpha[j, h] = exp(s - max_j s) / sum_j exp(s - max_j s), per head."""
    M = s.max(axis=0, keepdims=True)
    e = np.exp(s - M)
    return e / e.sum(axis=0, keepdims=True)


def head_of_channel(C: int, H: int) -> np.ndarray:
    return (np.arange(C) * H) // C


def aggregate(q, k, hp, nbrs: Sequence[np.ndarray], targets: Optional[Sequence[int]] = None):
    """m_i = sum_{j in N(i)} alpha_ij^{head(c)} h'_j for each target i ([EX] §3.1 step 2).

    nbrs[t] lists the neighbours of targets[t] (default: target t = atom t).
    Returns [len(nbrs), D, C] float64.
    """
    hp = np.asarray(hp, dtype=np.float64)
    N, D, C = hp.shape
    H = q.shape[1]
    hc = head_of_channel(C, H)
    targets = range(len(nbrs)) if targets is None else targets
    out = np.zeros((len(nbrs), D, C))
    for t, (i, js) in enumerate(zip(targets, nbrs)):
        js = np.asarray(js, dtype=np.int64)
        if js.size == 0:
            continue
        a = softmax_two_pass(logits(q[i], k[js]))       # [J, H]
        out[t] = np.einsum("jc,jdc->dc", a[:, hc], hp[js])
    return out


def forward(h, pos, q, k, w1, w2, lmax: int, nbrs: Sequence[np.ndarray],
            targets: Optional[Sequence[int]] = None, store=None) -> np.ndarray:
    """^h for each target: source coupling -> attention -> target coupling.

    Only the atoms that some target needs are coupled at the source.  store,
    if given, is applied to h' between the source coupling and the attention
    (``storage.round_bf16`` models the bf16 storage of h' that the bf16
    workloads specify); None keeps h' in float64.
    """
    N = np.asarray(h).shape[0]
    targets = list(range(N)) if targets is None else list(targets)
    need = np.unique(np.concatenate([np.asarray(j, dtype=np.int64) for j in nbrs] +
                                    [np.zeros(0, dtype=np.int64)]))
    hp = np.zeros(np.asarray(h).shape)
    if need.size:
        hp[need] = source_coupling(np.asarray(h)[need], np.asarray(pos)[need], w1, lmax)
        if store is not None:
            hp[need] = store(hp[need])
    m = aggregate(q, k, hp, nbrs, targets)
    return target_coupling(m, np.asarray(pos)[targets], w2, lmax)
