"""Pin the oracle's dense tensor product against EAAS (CPU only).

"E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §2.3 (Proposition 4.3)
states that the SO(3) tensor product of a feature with the geometric
encoding equals: rotate the feature into the frame whose z axis is r, apply
the sparse re-index of §2.2 (m_i = m_o for even ℓi+ℓf+ℓo, m_i = -m_o with a
sign for odd), and rotate back — with zero error.  This file writes that
sparse algorithm out independently of the oracle's dense sum, taking its
factors straight from sympy's Clebsch–Gordan coefficients, and requires the
two to agree to 1e-10 in float64, for every path up to ℓ = 3, random roll
angles about the aligned axis, r parallel to -z and r = 0.
"""
import numpy as np
import pytest
from sympy.physics.wigner import clebsch_gordan

from oracle import so3
from oracle.attention import tensor_product

RNG = np.random.default_rng(77)


def _axis_factor(li, lf, lo, mo):
    """(source m_i, factor) of output component m_o in the aligned frame."""
    if sum((li, lf, lo)) % 2 == 0:
        if abs(mo) > li:
            return None
        return mo, float(clebsch_gordan(li, lf, lo, mo, 0, mo))
    if mo == 0 or abs(mo) > li:
        return None
    return -mo, np.sign(mo) * float(clebsch_gordan(li, lf, lo, abs(mo), 0, abs(mo)))


def eaas_path(x, r, li, lf, lo, roll=0.0):
    """x [2li+1, C] -> [2lo+1, C] for one path by rotate / re-index / rotate back."""
    Q = so3.alignment_rotation(r) @ so3.rot_z(roll)
    xt = so3.wigner_D(li, Q).T @ x
    t = np.zeros((2 * lo + 1, x.shape[1]))
    for mo in range(-lo, lo + 1):
        f = _axis_factor(li, lf, lo, mo)
        if f is not None:
            t[mo + lo] = f[1] * xt[f[0] + li]
    t *= np.linalg.norm(r) ** lf
    return so3.wigner_D(lo, Q) @ t


R_CASES = [RNG.standard_normal(3) * 3, RNG.standard_normal(3) * 0.5,
           np.array([0.0, 0.0, -2.5]), np.array([0.0, 0.0, 1.7]), np.zeros(3)]


@pytest.mark.parametrize("path", so3.paths(3))
def test_eaas_equals_dense_per_path(path):
    li, lf, lo = path
    plist = so3.paths(3)
    C = 5
    for r in R_CASES:
        x = RNG.standard_normal((16, C))
        w = np.zeros((len(plist), C))
        w[plist.index(path)] = 1.0
        dense = tensor_product(x[None], r[None], w, 3)[0, lo * lo:(lo + 1) ** 2]
        for roll in (0.0, 1.234, -2.9):
            got = eaas_path(x[li * li:(li + 1) ** 2], r, li, lf, lo, roll)
            scale = max(1.0, np.abs(dense).max())
            assert np.abs(got - dense).max() < 1e-10 * scale, (path, r, roll)


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_eaas_equals_dense_weighted_sum(lmax):
    plist = so3.paths(lmax)
    C, N = 7, 4
    D = (lmax + 1) ** 2
    x = RNG.standard_normal((N, D, C))
    pos = RNG.standard_normal((N, 3)) * 4
    w = RNG.standard_normal((len(plist), C))
    dense = tensor_product(x, pos, w, lmax)
    for n in range(N):
        acc = np.zeros((D, C))
        for p, (li, lf, lo) in enumerate(plist):
            acc[lo * lo:(lo + 1) ** 2] += w[p] * eaas_path(
                x[n, li * li:(li + 1) ** 2], pos[n], li, lf, lo, roll=0.3 * n)
        assert np.abs(acc - dense[n]).max() < 1e-10 * max(1.0, np.abs(dense[n]).max())
