"""Backward pass of the oracle's forward (``attention.forward``).  Test
infrastructure only.

The pages name the backward pass as the step after the forward: the
Conservative mode takes forces as gradients of the energy, and the streaming
attention is recomputed rather than storing the attention weights
([EX] §3.2 on linear activation memory; [TS] §2.2).  This module writes out
the gradients of a scalar loss L = sum_i <G_i, ^h_i> (G the upstream
gradient) with respect to the features h, queries q and keys k, each step as
the plain adjoint of the corresponding forward step:

1. target coupling  ^h_i = T(m_i; r_i, w2) is linear in m_i, so
   dL/dm_i = T^*(G_i; r_i, w2), the transpose of the same dense contraction;
2. aggregation m_i = sum_j alpha_ij h'_j over the head of each channel:
   dL/dh'_j   += alpha_ij dL/dm_i                (over the targets i of j),
   dalpha_ij  = sum over the head's channels and components of
                dL/dm_i * h'_j,
   ds_ij      = alpha_ij (dalpha_ij - sum_j' alpha_ij' dalpha_ij')
                (softmax Jacobian),
   dL/dq_i    = sum_j ds_ij k_j / sqrt(d_k),
   dL/dk_j   += ds_ij q_i / sqrt(d_k);
3. source coupling h'_j = T(h_j; r_j, w1): dL/dh_j = T^*(dL/dh'_j; r_j, w1).

Positions enter only through the solid harmonics R(r) of the two couplings
(the logits are invariant scalars and the neighbour lists are piecewise
constant), so the position gradient is

   dL/dr_a = sum_c sum_p w2[p][c] sum T_p[m,mi,mf] G_a^{lo}[m][c] m_a^{li}[mi][c] dR^{lf}_{mf}(r_a)/dr_a
           + sum_c sum_p w1[p][c] sum T_p[m,mi,mf] dh'_a^{lo}[m][c] h_a^{li}[mi][c] dR^{lf}_{mf}(r_a)/dr_a

with the exact gradient of the solid harmonics (``so3.solid_harmonics_grad``);
forces are its negative.  Gradients with respect to the coupling weights are
not computed here.  Layouts as in ``attention``; every atom is a target
(nbrs[i] = N(i)).
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from . import so3
from .attention import _block, aggregate, head_of_channel, logits, softmax_two_pass, source_coupling


def tensor_product_adjoint(g: np.ndarray, pos: np.ndarray, w: np.ndarray, lmax: int) -> np.ndarray:
    """The transpose of ``attention.tensor_product`` as a linear map x -> y for
    fixed positions and weights:

        x^{li}[mi][c] = sum_{p=(li,lf,lo)} w[p][c] sum_{m,mf} T_p[m,mi,mf] g^{lo}[m][c] R^{lf}_{mf}(r).

    g [N, D, C]; pos [N, 3]; w [P, C].  Returns [N, D, C] float64.
    """
    g = np.asarray(g, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    plist = so3.paths(lmax)
    assert w.shape[0] == len(plist)
    R = [so3.solid_harmonics(l, pos) for l in range(lmax + 1)]
    x = np.zeros_like(g)
    for p, (li, lf, lo) in enumerate(plist):
        T = so3.real_cg(li, lf, lo)
        contrib = np.einsum("oif,noc,nf->nic", T, _block(g, lo), R[lf])
        x[:, li * li:(li + 1) * (li + 1), :] += contrib * w[p][None, None, :]
    return x


def attention_backward(q, k, hp, dm, nbrs: Sequence[np.ndarray]) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Step 2's adjoint: given dL/dm for every target, returns (dL/dh', dL/dq, dL/dk)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    hp = np.asarray(hp, dtype=np.float64)
    dm = np.asarray(dm, dtype=np.float64)
    N, D, C = hp.shape
    H, dk_ = q.shape[1], q.shape[2]
    hc = head_of_channel(C, H)
    member = np.zeros((C, H))
    member[np.arange(C), hc] = 1.0                  # channel -> head
    scale = 1.0 / np.sqrt(dk_)
    dhp = np.zeros_like(hp)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    for i, js in enumerate(nbrs):
        js = np.asarray(js, dtype=np.int64)
        if js.size == 0:
            continue
        a = softmax_two_pass(logits(q[i], k[js]))            # [J, H]
        da = np.einsum("dc,jdc->jc", dm[i], hp[js]) @ member   # [J, H]
        ds = a * (da - (a * da).sum(axis=0, keepdims=True))
        dq[i] += np.einsum("jh,jhd->hd", ds, k[js]) * scale
        np.add.at(dk, js, np.einsum("jh,hd->jhd", ds, q[i]) * scale)
        np.add.at(dhp, js, np.einsum("jc,dc->jdc", a[:, hc], dm[i]))
    return dhp, dq, dk


def attention_backward_at(q, k, hp, dm, nbrs, atoms):
    """``attention_backward`` evaluated at chosen atoms only, for systems too
    large to differentiate whole.

    For every a in ``atoms``: dL/dq_a (a as a target) and dL/dk_a, dL/dh'_a (a
    as a source, summed over the targets whose lists hold it).  ``nbrs`` maps
    an atom i to N(i) (a dict, or a sequence over all atoms) and must hold
    every atom in ``atoms`` and every target whose list holds one of them;
    ``hp`` and ``dm`` are read only at the atoms those lists touch.  Returns
    (dhp [len(atoms), D, C], dq [len(atoms), H, dk], dk [len(atoms), H, dk]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    C = hp.shape[2]
    H, dk_ = q.shape[1], q.shape[2]
    hc = head_of_channel(C, H)
    member = np.zeros((C, H))
    member[np.arange(C), hc] = 1.0
    scale = 1.0 / np.sqrt(dk_)
    row_cache = {}

    def target_terms(i):
        # alpha_i. and ds_i. over N(i) (the softmax backward of target i)
        if i not in row_cache:
            js = np.asarray(nbrs[i], dtype=np.int64)
            if js.size == 0:
                row_cache[i] = (js, None, None)
            else:
                a = softmax_two_pass(logits(q[i], k[js]))
                da = np.einsum("dc,jdc->jc", np.asarray(dm[i], np.float64),
                               np.asarray(hp[js], np.float64)) @ member
                row_cache[i] = (js, a, a * (da - (a * da).sum(axis=0, keepdims=True)))
        return row_cache[i]

    holders = {}
    keys = nbrs.keys() if isinstance(nbrs, dict) else range(len(nbrs))
    wanted = set(int(a) for a in atoms)
    for i in keys:
        for j in np.asarray(nbrs[i], dtype=np.int64):
            if int(j) in wanted:
                holders.setdefault(int(j), []).append(int(i))
    A = len(atoms)
    dhp = np.zeros((A,) + hp.shape[1:])
    dq = np.zeros((A, H, dk_))
    dk = np.zeros((A, H, dk_))
    for t, a_ in enumerate(atoms):
        js, a, ds = target_terms(int(a_))
        if js.size:
            dq[t] = np.einsum("jh,jhd->hd", ds, k[js]) * scale
        for i in holders.get(int(a_), []):
            js, a, ds = target_terms(i)
            for pos_in_row in np.nonzero(js == int(a_))[0]:
                dk[t] += np.einsum("h,hd->hd", ds[pos_in_row], q[i]) * scale
                dhp[t] += a[pos_in_row][hc][None, :] * np.asarray(dm[i], np.float64)
    return dhp, dq, dk


def backward(h, pos, q, k, w1, w2, lmax: int, nbrs: Sequence[np.ndarray],
             G) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(dL/dh, dL/dq, dL/dk) for L = sum_i <G_i, ^h_i>, ^h = attention.forward."""
    pos = np.asarray(pos, dtype=np.float64)
    hp = source_coupling(h, pos, w1, lmax)
    dm = tensor_product_adjoint(G, pos, w2, lmax)
    dhp, dq, dk = attention_backward(q, k, hp, dm, nbrs)
    dh = tensor_product_adjoint(dhp, pos, w1, lmax)
    return dh, dq, dk


def coupling_position_grad(g, x, pos, w, lmax: int) -> np.ndarray:
    """d<g, T(x; r, w)>/dr for each atom: [N, 3].

    sum_c sum_p w[p][c] sum_{m,mi,mf} T_p[m,mi,mf] g^{lo}[m][c] x^{li}[mi][c] dR^{lf}_{mf}/dr.
    """
    g = np.asarray(g, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    dR = [so3.solid_harmonics_grad(l, pos) for l in range(lmax + 1)]    # [N, 2l+1, 3]
    out = np.zeros((pos.shape[0], 3))
    for p, (li, lf, lo) in enumerate(so3.paths(lmax)):
        if lf == 0:
            continue
        T = so3.real_cg(li, lf, lo)
        bil = np.einsum("oif,noc,nic,c->nf", T, _block(g, lo), _block(x, li), w[p])
        out += np.einsum("nf,nfa->na", bil, dR[lf])
    return out


def position_grad(h, pos, q, k, w1, w2, lmax: int, nbrs: Sequence[np.ndarray], G) -> np.ndarray:
    """dL/dr [N, 3] for L = sum_i <G_i, ^h_i> (forces are -dL/dr)."""
    pos = np.asarray(pos, dtype=np.float64)
    hp = source_coupling(h, pos, w1, lmax)
    m = aggregate(q, k, hp, nbrs)
    dm = tensor_product_adjoint(G, pos, w2, lmax)
    dhp, _, _ = attention_backward(q, k, hp, dm, nbrs)
    return (coupling_position_grad(G, m, pos, w2, lmax)
            + coupling_position_grad(dhp, h, pos, w1, lmax))
