"""Pins of the oracle's edge-centric eSCN convolution (oracle/escn.py).

"EquiformerV3: Scaling Efficient, Expressive, and General SE(3)-Equivariant Graph Attention Transformers", section "eSCN卷积与SO(2)线性层": rotate by D_ij,
apply an SO(2) linear layer within each degree's components, rotate back.
A plausible mistake (a transposed rotation, a wrong sign in the +-m blocks, a
mixed-up weight row, the wrong edge direction) fails one of:

* identity weights (W0 = W1 = delta, W2 = 0, M_max = L): the message is h_j
  itself, so out_i = sum_j h_j — independent of every rotation;
* the m = 0 projector (W0 = delta, nothing else): degree 0 passes unchanged and
  degree 1 gives sum_j (r^_ij . h_j) r^_ij, written out with the (y, z, x)
  order of the real degree-1 basis — a closed form with no Wigner-D matrix;
* a random roll about each edge axis (Q_ij R_z(gamma)) changes nothing: the
  [[W1, -W2], [W2, W1]] blocks commute with rotations about z (a symmetric
  block, or a transposed one with the wrong sign, would not);
* rotating positions about the origin and features by D(G) rotates the output.
"""
import numpy as np
import pytest

from oracle import so3
from oracle.escn import escn_conv, num_weights, weight_rows
from oracle.graph import radius_graph
from equivariant_graph_attention_b200 import synth

RNG = np.random.default_rng(23)


def _system(L=2, C=5, n=14, seed=4):
    wl = synth.small_cube(n, 5.0, 3.2, 16, L, C, 1, 8, "f32")
    d = synth.make(wl, seed=seed)
    nbrs, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    return wl, d, nbrs


def _identity_weights(L, mmax, C):
    w = np.zeros((num_weights(L, mmax), C))
    w0, blocks = weight_rows(L, mmax)
    for l in range(L + 1):
        w[w0[l, l]] = 1.0
    for m, (w1, _) in enumerate(blocks, start=1):
        for l in range(m, L + 1):
            w[w1[l - m, l - m]] = 1.0
    return w


def test_weight_count():
    assert num_weights(2, 2) == 9 + 2 * 4 + 2 * 1
    assert num_weights(3, 1) == 16 + 2 * 9
    assert num_weights(1, 0) == 4


@pytest.mark.parametrize("L", [1, 2, 3])
def test_identity_weights_sum_the_neighbours(L):
    wl, d, nbrs = _system(L=L)
    out = escn_conv(d["h"], d["pos"], _identity_weights(L, L, wl.C), L, L, nbrs)
    want = np.array([np.asarray(d["h"], np.float64)[js].sum(axis=0) for js in nbrs])
    assert np.max(np.abs(out - want)) < 1e-12 * np.max(np.abs(want))


def test_m0_projector_closed_form():
    L = 1
    wl, d, nbrs = _system(L=L)
    w = np.zeros((num_weights(L, 0), wl.C))
    w0, _ = weight_rows(L, 0)
    w[w0[0, 0]] = 1.0
    w[w0[1, 1]] = 1.0
    out = escn_conv(d["h"], d["pos"], w, L, 0, nbrs)
    h = np.asarray(d["h"], np.float64)
    pos = np.asarray(d["pos"], np.float64)
    for i, js in enumerate(nbrs):
        want0 = h[js, 0].sum(axis=0)
        want1 = np.zeros((3, wl.C))
        for j in js:
            r = pos[j] - pos[i]
            u = (r / np.linalg.norm(r))[[1, 2, 0]]           # (y, z, x)
            want1 += np.outer(u, u @ h[j, 1:4])
        assert np.allclose(out[i, 0], want0, atol=1e-12)
        assert np.allclose(out[i, 1:4], want1, atol=1e-12)


@pytest.mark.parametrize("L,mmax", [(2, 2), (3, 1), (3, 3)])
def test_independent_of_the_roll(L, mmax):
    wl, d, nbrs = _system(L=L)
    w = RNG.standard_normal((num_weights(L, mmax), wl.C))
    a = escn_conv(d["h"], d["pos"], w, L, mmax, nbrs)
    b = escn_conv(d["h"], d["pos"], w, L, mmax, nbrs, roll=lambda i, j: 0.37 * i + 1.1 * j + 0.2)
    assert np.max(np.abs(a - b)) < 1e-10 * np.max(np.abs(a))
    # a symmetric +-m block would depend on the roll: the pin has teeth
    import oracle.escn as E
    orig = E.so2_linear

    def sym(xt, w, L, mmax):
        y = orig(xt, w, L, 0)
        _, blocks = weight_rows(L, mmax)
        comp = lambda l, m: l * l + l + m
        for lo in range(L + 1):
            for li in range(L + 1):
                for m in range(1, min(mmax, lo, li) + 1):
                    w1, w2 = w[blocks[m - 1][0][lo - m, li - m]], w[blocks[m - 1][1][lo - m, li - m]]
                    xp, xm = xt[comp(li, m)], xt[comp(li, -m)]
                    y[comp(lo, m)] += w1 * xp + w2 * xm
                    y[comp(lo, -m)] += w2 * xp + w1 * xm
        return y
    E.so2_linear = sym
    try:
        c = escn_conv(d["h"], d["pos"], w, L, mmax, nbrs)
        e = escn_conv(d["h"], d["pos"], w, L, mmax, nbrs, roll=lambda i, j: 0.37 * i + 1.1 * j + 0.2)
    finally:
        E.so2_linear = orig
    assert np.max(np.abs(c - e)) > 1e-3 * np.max(np.abs(c))


@pytest.mark.parametrize("L", [1, 2, 3])
def test_rotation_equivariance(L):
    wl, d, nbrs = _system(L=L)
    w = RNG.standard_normal((num_weights(L, L), wl.C))
    G = so3.alignment_rotation(RNG.standard_normal(3)) @ so3.rot_z(0.61)
    Ds = [so3.wigner_D(l, G) for l in range(L + 1)]

    def rot(x):
        y = np.array(x, dtype=np.float64)
        for l in range(L + 1):
            y[:, l * l:(l + 1) ** 2] = np.einsum("ab,nbc->nac", Ds[l], y[:, l * l:(l + 1) ** 2])
        return y
    out = escn_conv(d["h"], d["pos"], w, L, L, nbrs)
    out_r = escn_conv(rot(d["h"]), np.asarray(d["pos"], np.float64) @ G.T, w, L, L, nbrs)
    assert np.max(np.abs(out_r - rot(out))) < 1e-10 * np.max(np.abs(out))
