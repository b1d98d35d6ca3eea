"""Pins for the oracle's SO(3) building blocks (CPU only).

Each check compares the oracle with something other than itself: a library
routine (sympy's Clebsch–Gordan coefficients, scipy's spherical harmonics), a
textbook closed form, or an invariant that the mathematics fixes.  Pages:
[EX] "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构",
[TS] "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation Memory".
"""
import numpy as np
import pytest
import scipy.special
from sympy.physics.wigner import clebsch_gordan

from oracle import so3
from equivariant_graph_attention_b200 import synth

RNG = np.random.default_rng(2024)
PERM = np.array([[0, 1, 0], [0, 0, 1], [1, 0, 0]], dtype=float)   # (x,y,z) -> (y,z,x)


def _rand_rot():
    a = RNG.standard_normal((3, 3))
    q, r = np.linalg.qr(a)
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


# ---------------------------------------------------------------- Clebsch–Gordan
def test_cg_matches_sympy_all_l_le_4():
    worst = 0.0
    for j1 in range(5):
        for j2 in range(5):
            for J in range(abs(j1 - j2), min(j1 + j2, 6) + 1):
                for m1 in range(-j1, j1 + 1):
                    for m2 in range(-j2, j2 + 1):
                        M = m1 + m2
                        if abs(M) > J:
                            continue
                        ref = float(clebsch_gordan(j1, j2, J, m1, m2, M))
                        worst = max(worst, abs(so3.cg_complex(j1, m1, j2, m2, J, M) - ref))
    assert worst < 1e-14


def test_cg_selection_zeros():
    assert so3.cg_complex(1, 1, 1, 0, 2, 0) == 0.0        # M != m1 + m2
    assert so3.cg_complex(1, 0, 1, 0, 3, 0) == 0.0        # triangle violated
    assert so3.cg_complex(1, 0, 1, 0, 1, 0) == 0.0        # <1 0;1 0|1 0> vanishes (odd sum)


# ---------------------------------------------------------------- harmonics
def test_real_basis_unitary():
    for l in range(5):
        U = so3.real_basis(l)
        assert np.allclose(U @ U.conj().T, np.eye(2 * l + 1), atol=1e-15)


@pytest.mark.parametrize("l", [0, 1, 2, 3, 4])
def test_complex_sph_harm_matches_scipy(l):
    u = RNG.standard_normal((50, 3))
    r = np.linalg.norm(u, axis=1)
    theta = np.arccos(u[:, 2] / r)
    phi = np.arctan2(u[:, 1], u[:, 0])
    got = so3.sph_harm_complex(l, u)
    for m in range(-l, l + 1):
        ref = scipy.special.sph_harm_y(l, m, theta, phi)
        assert np.max(np.abs(got[:, m + l] - ref)) < 1e-13


def _real_table(l, u):
    """Textbook real spherical harmonics (standard table, Condon–Shortley phase
    cancelled), written as polynomials in x, y, z on the unit sphere."""
    x, y, z = (u / np.linalg.norm(u, axis=1, keepdims=True)).T
    pi = np.pi
    if l == 1:
        c = np.sqrt(3 / (4 * pi))
        return np.stack([c * y, c * z, c * x], 1)
    if l == 2:
        return np.stack([0.5 * np.sqrt(15 / pi) * x * y,
                         0.5 * np.sqrt(15 / pi) * y * z,
                         0.25 * np.sqrt(5 / pi) * (3 * z * z - 1),
                         0.5 * np.sqrt(15 / pi) * x * z,
                         0.25 * np.sqrt(15 / pi) * (x * x - y * y)], 1)
    if l == 3:
        return np.stack([0.25 * np.sqrt(35 / (2 * pi)) * y * (3 * x * x - y * y),
                         0.5 * np.sqrt(105 / pi) * x * y * z,
                         0.25 * np.sqrt(21 / (2 * pi)) * y * (5 * z * z - 1),
                         0.25 * np.sqrt(7 / pi) * (5 * z ** 3 - 3 * z),
                         0.25 * np.sqrt(21 / (2 * pi)) * x * (5 * z * z - 1),
                         0.25 * np.sqrt(105 / pi) * (x * x - y * y) * z,
                         0.25 * np.sqrt(35 / (2 * pi)) * x * (x * x - 3 * y * y)], 1)
    raise ValueError


@pytest.mark.parametrize("l", [1, 2, 3])
def test_real_sph_harm_textbook_table(l):
    u = RNG.standard_normal((40, 3))
    assert np.max(np.abs(so3.sph_harm_real(l, u) - _real_table(l, u))) < 1e-13


def test_solid_harmonics_degree1_is_yzx():
    r = RNG.standard_normal((20, 3)) * 4
    assert np.allclose(so3.solid_harmonics(1, r), r[:, [1, 2, 0]], atol=1e-13)


@pytest.mark.parametrize("l", [0, 1, 2, 3])
def test_solid_harmonics_aligned_sparsity_lemma(l):
    # [TS] §2.1 (Lemma 4.1): in the frame whose z axis is r only m = 0 is nonzero
    for s in [0.3, 1.0, 7.5]:
        R = so3.solid_harmonics(l, np.array([[0.0, 0.0, s]]))[0]
        e = np.zeros(2 * l + 1)
        e[l] = s ** l
        assert np.allclose(R, e, atol=1e-13 * max(1, s ** l))
    R = so3.solid_harmonics(l, np.array([[0.0, 0.0, -2.0]]))[0]   # r parallel to -z
    e = np.zeros(2 * l + 1)
    e[l] = (-2.0) ** l
    assert np.allclose(R, e, atol=1e-12)


@pytest.mark.parametrize("l", [0, 1, 2, 3])
def test_solid_harmonics_addition_theorem_and_homogeneity(l):
    r = RNG.standard_normal((30, 3)) * 3
    R = so3.solid_harmonics(l, r)
    n = np.linalg.norm(r, axis=1)
    assert np.allclose(np.sum(R * R, 1), n ** (2 * l), rtol=1e-12)
    assert np.allclose(so3.solid_harmonics(l, 2.5 * r), 2.5 ** l * R, rtol=1e-12)


def test_solid_harmonics_at_origin():
    z = np.zeros((1, 3))
    assert np.array_equal(so3.solid_harmonics(0, z), np.ones((1, 1)))
    for l in (1, 2, 3):
        assert np.array_equal(so3.solid_harmonics(l, z), np.zeros((1, 2 * l + 1)))


# ---------------------------------------------------------------- rotations
def test_alignment_rotation_properties():
    cases = [RNG.standard_normal(3) for _ in range(20)] + [
        np.array([0.0, 0.0, 3.0]), np.array([0.0, 0.0, -3.0]), np.array([1e-9, 0.0, -1.0])]
    for r in cases:
        Q = so3.alignment_rotation(r)
        assert np.allclose(Q @ np.array([0, 0, 1.0]), r / np.linalg.norm(r), atol=1e-12)
        assert np.allclose(Q.T @ Q, np.eye(3), atol=1e-12)
        # [EX] §5.2 asks det R ≈ 1; held here to 1e-12
        assert abs(np.linalg.det(Q) - 1.0) < 1e-12
    assert np.array_equal(so3.alignment_rotation(np.zeros(3)), np.eye(3))


@pytest.mark.parametrize("l", [0, 1, 2, 3])
def test_wigner_D_representation(l):
    Q1, Q2 = _rand_rot(), _rand_rot()
    D1, D2 = so3.wigner_D(l, Q1), so3.wigner_D(l, Q2)
    assert np.allclose(D1 @ D1.T, np.eye(2 * l + 1), atol=1e-12)
    assert abs(np.linalg.det(D1) - 1.0) < 1e-12
    assert np.allclose(so3.wigner_D(l, Q1 @ Q2), D1 @ D2, atol=1e-12)
    u = RNG.standard_normal((25, 3))     # fresh points, not the fit directions
    if l:
        assert np.allclose(so3.sph_harm_real(l, u @ Q1.T), so3.sph_harm_real(l, u) @ D1.T,
                           atol=1e-12)


def test_wigner_D1_is_permuted_rotation():
    Q = _rand_rot()
    assert np.allclose(so3.wigner_D(1, Q), PERM @ Q @ PERM.T, atol=1e-13)


# ---------------------------------------------------------------- coupling tensors
def test_paths_counts_and_fan_in():
    fan = {1: [2, 3], 2: [3, 6, 6], 3: [4, 9, 11, 10]}
    for lmax, total in [(1, 5), (2, 15), (3, 34)]:
        p = so3.paths(lmax)
        assert len(p) == total
        assert [sum(1 for t in p if t[2] == lo) for lo in range(lmax + 1)] == fan[lmax]
        odd = sum(1 for t in p if sum(t) % 2)
        assert odd == {1: 1, 2: 4, 3: 11}[lmax]
        # the generator orders weight rows the same way (interface agreement)
        assert p == synth.coupling_paths(lmax)


@pytest.mark.parametrize("path", so3.paths(3))
def test_real_cg_orthonormal_rows(path):
    T = so3.real_cg(*path)
    M = T.reshape(T.shape[0], -1)
    assert np.allclose(M @ M.T, np.eye(T.shape[0]), atol=1e-13)


@pytest.mark.parametrize("path", so3.paths(3))
def test_real_cg_equivariant(path):
    li, lf, lo = path
    T = so3.real_cg(*path)
    Q = _rand_rot()
    a, b = RNG.standard_normal(2 * li + 1), RNG.standard_normal(2 * lf + 1)
    lhs = np.einsum("oif,i,f->o", T, so3.wigner_D(li, Q) @ a, so3.wigner_D(lf, Q) @ b)
    rhs = so3.wigner_D(lo, Q) @ np.einsum("oif,i,f->o", T, a, b)
    assert np.allclose(lhs, rhs, atol=1e-12)


def test_real_cg_closed_forms():
    for l in range(4):
        assert np.allclose(so3.real_cg(0, l, l)[:, 0, :], np.eye(2 * l + 1), atol=1e-15)
        assert np.allclose(so3.real_cg(l, 0, l)[:, :, 0], np.eye(2 * l + 1), atol=1e-15)
    # (1,1 -> 0) is -(a . b)/sqrt3
    assert np.allclose(so3.real_cg(1, 1, 0)[0], -np.eye(3) / np.sqrt(3), atol=1e-15)
    # (1,1 -> 1) is (a x b)/sqrt2 in (y, z, x) components
    a, b = RNG.standard_normal(3), RNG.standard_normal(3)
    got = np.einsum("oif,i,f->o", so3.real_cg(1, 1, 1), PERM @ a, PERM @ b)
    assert np.allclose(got, PERM @ np.cross(a, b) / np.sqrt(2), atol=1e-14)


@pytest.mark.parametrize("path", so3.paths(3))
def test_real_cg_gaunt_closed_form(path):
    """Coupling a direction's harmonics with themselves gives the harmonic of
    the output degree: (R^li(r) x R^lf(r))^lo = <li 0; lf 0|lo 0> |r|^(li+lf-lo) R^lo(r)."""
    li, lf, lo = path
    r = RNG.standard_normal(3) * 2.0
    got = np.einsum("oif,i,f->o", so3.real_cg(*path),
                    so3.solid_harmonics(li, r[None])[0], so3.solid_harmonics(lf, r[None])[0])
    ref = (float(clebsch_gordan(li, lf, lo, 0, 0, 0)) * np.linalg.norm(r) ** (li + lf - lo)
           * so3.solid_harmonics(lo, r[None])[0])
    assert np.allclose(got, ref, atol=1e-12 * max(1.0, np.abs(ref).max()))


@pytest.mark.parametrize("path", so3.paths(3))
def test_real_cg_axis_slice_selection_rule(path):
    """[EX] §2.2 / [TS] Eq. 13: with m_f = 0 only m_i = m_o (even li+lf+lo) or
    m_i = -m_o with a sign (odd) survive.  The nonzero values are the complex
    coefficients <li m; lf 0|lo m> (sympy), times sgn(m_o) in the odd case."""
    li, lf, lo = path
    S = so3.real_cg(*path)[:, :, lf]
    ref = np.zeros_like(S)
    for mo in range(-lo, lo + 1):
        if sum(path) % 2 == 0:
            if abs(mo) <= li:
                ref[mo + lo, mo + li] = float(clebsch_gordan(li, lf, lo, mo, 0, mo))
        elif abs(mo) <= li and mo != 0:
            ref[mo + lo, -mo + li] = np.sign(mo) * float(
                clebsch_gordan(li, lf, lo, abs(mo), 0, abs(mo)))
    assert np.allclose(S, ref, atol=1e-14)
