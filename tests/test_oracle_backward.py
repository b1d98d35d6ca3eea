"""Pins of the oracle's backward pass (oracle/backward.py).

* The adjoint of the dense coupling is checked against the forward coupling
  through the defining identity <T x, g> = <x, T* g> on random x, g (no
  formula retyped: the forward is called as is).
* The whole backward (dL/dh, dL/dq, dL/dk) is checked against central finite
  differences of the oracle forward on a tiny system, where fp64 differences
  are accurate to about 1e-8.
* Two special cases: a zero upstream gradient gives zero gradients, and a
  target with a single neighbour (alpha = 1 identically) passes dL/dm straight
  to that neighbour's h' with no logit gradient.
* The evaluation at chosen atoms (attention_backward_at, for systems too
  large to differentiate whole) agrees with the whole-system attention
  backward at those atoms, whose neighbour lists are given as a dict holding
  only what it needs.
"""
import numpy as np
import pytest

from oracle import so3
from oracle.attention import forward, tensor_product
from oracle.backward import (attention_backward, attention_backward_at, backward, position_grad,
                             tensor_product_adjoint)
from oracle.graph import radius_graph


def _system(seed, n=10, lmax=2, C=8, H=2, dk=4):
    rng = np.random.default_rng(seed)
    D = (lmax + 1) ** 2
    P = len(so3.paths(lmax))
    pos_q = rng.integers(-3 << 16, 3 << 16, size=(n, 3), dtype=np.int64)
    pos = pos_q * 2.0 ** -16
    h = rng.standard_normal((n, D, C))
    q = rng.standard_normal((n, H, dk))
    k = rng.standard_normal((n, H, dk))
    w1 = rng.standard_normal((P, C)) / np.sqrt(3)
    w2 = rng.standard_normal((P, C)) / np.sqrt(3)
    lists, _ = radius_graph(pos_q.astype(np.int32), 4 << 16, K=6)
    G = rng.standard_normal((n, D, C))
    return dict(h=h, pos=pos, q=q, k=k, w1=w1, w2=w2, lmax=lmax, nbrs=lists, G=G)


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_adjoint_identity(lmax):
    rng = np.random.default_rng(lmax)
    D = (lmax + 1) ** 2
    x = rng.standard_normal((5, D, 6))
    g = rng.standard_normal((5, D, 6))
    pos = rng.standard_normal((5, 3)) * 2
    w = rng.standard_normal((len(so3.paths(lmax)), 6))
    lhs = np.sum(tensor_product(x, pos, w, lmax) * g)
    rhs = np.sum(x * tensor_product_adjoint(g, pos, w, lmax))
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs))


def _loss(s, **over):
    a = dict(s, **over)
    out = forward(a["h"], a["pos"], a["q"], a["k"], a["w1"], a["w2"], a["lmax"], a["nbrs"])
    return float(np.sum(out * a["G"]))


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_matches_finite_differences(seed):
    s = _system(seed)
    dh, dq, dk = backward(s["h"], s["pos"], s["q"], s["k"], s["w1"], s["w2"], s["lmax"],
                          s["nbrs"], s["G"])
    rng = np.random.default_rng(100 + seed)
    eps = 1e-5
    for name, grad in (("h", dh), ("q", dq), ("k", dk)):
        arr = s[name]
        for _ in range(12):
            idx = tuple(int(rng.integers(0, m)) for m in arr.shape)
            up, dn = arr.copy(), arr.copy()
            up[idx] += eps
            dn[idx] -= eps
            fd = (_loss(s, **{name: up}) - _loss(s, **{name: dn})) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * (1.0 + abs(fd)), (name, idx, fd, grad[idx])


def test_zero_upstream_gradient_gives_zero():
    s = _system(3)
    dh, dq, dk = backward(s["h"], s["pos"], s["q"], s["k"], s["w1"], s["w2"], s["lmax"],
                          s["nbrs"], np.zeros_like(s["G"]))
    assert not dh.any() and not dq.any() and not dk.any()


def test_single_neighbour_has_no_logit_gradient():
    """With one neighbour alpha = 1 identically, so dL/dq and dL/dk vanish and
    dL/dh' is dL/dm of the target."""
    rng = np.random.default_rng(5)
    N, D, C, H, dk = 2, 4, 4, 2, 4
    hp = rng.standard_normal((N, D, C))
    q = rng.standard_normal((N, H, dk))
    k = rng.standard_normal((N, H, dk))
    dm = rng.standard_normal((N, D, C))
    nbrs = [np.array([1]), np.array([], dtype=np.int64)]
    dhp, dq, dk_ = attention_backward(q, k, hp, dm, nbrs)
    assert np.allclose(dq, 0.0, atol=1e-14) and np.allclose(dk_, 0.0, atol=1e-14)
    assert np.allclose(dhp[1], dm[0]) and not dhp[0].any()


@pytest.mark.parametrize("l", [1, 2, 3])
def test_solid_harmonics_gradient_matches_finite_differences(l):
    rng = np.random.default_rng(l)
    r = rng.standard_normal((6, 3)) * 1.7
    got = so3.solid_harmonics_grad(l, r)
    eps = 1e-6
    for a in range(3):
        e = np.zeros(3)
        e[a] = eps
        fd = (so3.solid_harmonics(l, r + e) - so3.solid_harmonics(l, r - e)) / (2 * eps)
        assert np.allclose(got[..., a], fd, rtol=1e-7, atol=1e-7 * (1 + np.abs(fd).max()))


def test_solid_harmonics_gradient_closed_form_degree1():
    """Degree 1 is linear: R^1 = (y, z, x) in the basis order, so its gradient
    is a constant permutation matrix."""
    g = so3.solid_harmonics_grad(1, np.array([[0.3, -1.2, 2.5]]))[0]
    assert np.allclose(g, [[0, 1, 0], [0, 0, 1], [1, 0, 0]], atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1])
def test_position_gradient_matches_finite_differences(seed):
    """dL/dr against central differences of the oracle forward in the
    positions (neighbour lists held fixed, as the gradient assumes)."""
    s = _system(seed)
    grad = position_grad(s["h"], s["pos"], s["q"], s["k"], s["w1"], s["w2"], s["lmax"],
                         s["nbrs"], s["G"])
    eps = 1e-6
    for a in range(s["pos"].shape[0]):
        for c in range(3):
            up, dn = s["pos"].copy(), s["pos"].copy()
            up[a, c] += eps
            dn[a, c] -= eps
            fd = (_loss(s, pos=up) - _loss(s, pos=dn)) / (2 * eps)
            assert abs(fd - grad[a, c]) <= 1e-5 * (1.0 + abs(fd)), (a, c, fd, grad[a, c])


def test_backward_at_chosen_atoms_matches_whole_system():
    rng = np.random.default_rng(11)
    n, D, C, H, dk = 40, 4, 8, 2, 4
    pos_q = rng.integers(-4 << 16, 4 << 16, size=(n, 3), dtype=np.int64).astype(np.int32)
    lists, _ = radius_graph(pos_q, 3 << 16, K=7)
    q = rng.standard_normal((n, H, dk))
    k = rng.standard_normal((n, H, dk))
    hp = rng.standard_normal((n, D, C))
    dm = rng.standard_normal((n, D, C))
    dhp, dq, dk_ = attention_backward(q, k, hp, dm, lists)
    atoms = [0, 7, 19, n - 1]
    need = set(atoms) | {i for i in range(n) if set(lists[i].tolist()) & set(atoms)}
    sub = {i: lists[i] for i in need}
    a_dhp, a_dq, a_dk = attention_backward_at(q, k, hp, dm, sub, atoms)
    assert np.abs(a_dhp - dhp[atoms]).max() <= 1e-12 * max(1.0, np.abs(dhp).max())
    assert np.abs(a_dq - dq[atoms]).max() <= 1e-12 * max(1.0, np.abs(dq).max())
    assert np.abs(a_dk - dk_[atoms]).max() <= 1e-12 * max(1.0, np.abs(dk_).max())
    assert np.abs(dk_[atoms]).max() > 0 and np.abs(dq[atoms]).max() > 0
