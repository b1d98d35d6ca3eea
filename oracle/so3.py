"""SO(3) building blocks of the oracle, in float64.  Test infrastructure only.

Conventions (the pages leave them open; these are the plainest readings):

* Complex spherical harmonics Y_l^m carry the Condon–Shortley phase.
* Real harmonics: for m > 0, Y_lm = (Y_l^{-m} + (-1)^m Y_l^m)/sqrt2; m = 0,
  Y_l0 = Y_l^0; m < 0, Y_lm = i (Y_l^m - (-1)^m Y_l^{-m})/sqrt2.  Components
  are ordered m = -l..l, so degree 1 is proportional to (y, z, x).
* Solid harmonics are Racah-normalised, R^l_m(r) = sqrt(4 pi/(2l+1)) |r|^l
  Y_lm(r^), so that R^l(|r| z^) = |r|^l e_0 — the "maximal sparsity" of
  [TS] §2.1 (Lemma 4.1) — and R^1(r) = (y, z, x).
* Real coupling tensor of path (li, lf, lo): the complex CG tensor moved to
  the real basis; it is real when li+lf+lo is even and purely imaginary when
  odd, and the odd case keeps the imaginary part ([EX] §2.2 treats both
  parities).
* Wigner-D matrices act on real components: Y_l(Q u) = D^l(Q) Y_l(u).
* The alignment rotation is Q = R_z(phi) R_y(theta) with (theta, phi) the polar
  angles of r, so Q z^ = r^ ([EX] §2.1 "compute_alignment_rotation").
"""
from __future__ import annotations

from fractions import Fraction
from functools import lru_cache
from math import factorial

import numpy as np


def comp(l: int, m: int) -> int:
    """Row of component (l, m) in the [ (lmax+1)^2 ] layout."""
    return l * l + l + m


# --------------------------------------------------------------------------
# Clebsch–Gordan coefficients (Racah's closed formula)
# --------------------------------------------------------------------------
def cg_complex(j1: int, m1: int, j2: int, m2: int, J: int, M: int) -> float:
    """<j1 m1; j2 m2 | J M> for integer angular momenta, Racah formula.

    The square root is taken of an exact rational, so the only rounding is the
    final conversion to float.
    """
    if M != m1 + m2:
        return 0.0
    if not (abs(j1 - j2) <= J <= j1 + j2):
        return 0.0
    if abs(m1) > j1 or abs(m2) > j2 or abs(M) > J:
        return 0.0
    f = factorial
    pre = Fraction((2 * J + 1) * f(J + j1 - j2) * f(J - j1 + j2) * f(j1 + j2 - J),
                   f(j1 + j2 + J + 1))
    pre *= f(J + M) * f(J - M) * f(j1 - m1) * f(j1 + m1) * f(j2 - m2) * f(j2 + m2)
    s = Fraction(0)
    for k in range(0, j1 + j2 - J + 1):
        args = [k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k]
        if min(args) < 0:
            continue
        den = 1
        for a in args:
            den *= f(a)
        s += Fraction((-1) ** k, den)
    # value = sqrt(pre) * s = sign(s) * sqrt(pre * s^2), the radicand exact
    if s == 0:
        return 0.0
    sign = 1.0 if s > 0 else -1.0
    return sign * float(np.sqrt(float(pre * s * s)))


# --------------------------------------------------------------------------
# Complex -> real basis change
# --------------------------------------------------------------------------
def real_basis(l: int) -> np.ndarray:
    """Unitary U (2l+1 x 2l+1) with Y_real[m] = sum_mu U[m, mu] Y_complex[mu]."""
    U = np.zeros((2 * l + 1, 2 * l + 1), dtype=np.complex128)
    r2 = 1.0 / np.sqrt(2.0)
    for m in range(-l, l + 1):
        a = m + l
        if m > 0:
            U[a, -m + l] = r2
            U[a, m + l] = (-1) ** m * r2
        elif m == 0:
            U[a, l] = 1.0
        else:
            U[a, m + l] = 1j * r2
            U[a, -m + l] = -1j * (-1) ** m * r2
    return U


# --------------------------------------------------------------------------
# Spherical harmonics
# --------------------------------------------------------------------------
def _legendre_assoc(l: int, m: int, x: np.ndarray) -> np.ndarray:
    """P_l^m(x), m >= 0, with Condon–Shortley phase, via Rodrigues' formula."""
    P = np.polynomial.Polynomial([-1.0, 0.0, 1.0]) ** l          # (x^2 - 1)^l
    P = P.deriv(l + m) / (2.0 ** l * factorial(l))
    return (-1) ** m * (1.0 - x * x) ** (m / 2.0) * P(x)


def sph_harm_complex(l: int, u: np.ndarray) -> np.ndarray:
    """Complex Y_l^mu(u^) for mu = -l..l; u [..., 3] nonzero. Returns [..., 2l+1]."""
    u = np.asarray(u, dtype=np.float64)
    r = np.linalg.norm(u, axis=-1)
    ct = u[..., 2] / r
    ct = np.clip(ct, -1.0, 1.0)
    phi = np.arctan2(u[..., 1], u[..., 0])
    out = np.zeros(u.shape[:-1] + (2 * l + 1,), dtype=np.complex128)
    for m in range(0, l + 1):
        norm = np.sqrt((2 * l + 1) / (4 * np.pi) * factorial(l - m) / factorial(l + m))
        y = norm * _legendre_assoc(l, m, ct) * np.exp(1j * m * phi)
        out[..., m + l] = y
        if m > 0:
            out[..., -m + l] = (-1) ** m * np.conj(y)
    return out


def sph_harm_real(l: int, u: np.ndarray) -> np.ndarray:
    """Real Y_lm(u^), m = -l..l, for nonzero u [..., 3]. Returns [..., 2l+1]."""
    yc = sph_harm_complex(l, u)
    yr = yc @ real_basis(l).T
    assert np.max(np.abs(yr.imag), initial=0.0) < 1e-12
    return yr.real


def solid_harmonics(l: int, r: np.ndarray) -> np.ndarray:
    """Racah-normalised real solid harmonics R^l(r) [..., 2l+1]; R^l(0) = delta_l0.

    [TS] §2.1 (Lemma 4.1): in the frame whose z axis is r only m = 0 survives.
    """
    r = np.asarray(r, dtype=np.float64)
    n = np.linalg.norm(r, axis=-1)
    out = np.zeros(r.shape[:-1] + (2 * l + 1,))
    if l == 0:
        out[...] = 1.0
        return out
    nz = n > 0
    if np.any(nz):
        out[nz] = (np.sqrt(4 * np.pi / (2 * l + 1)) * n[nz, None] ** l
                   * sph_harm_real(l, r[nz]))
    return out


_MONO_CACHE = {}


def _monomials(l: int):
    """Exponents (a, b, c), a + b + c = l, of the homogeneous monomials x^a y^b z^c."""
    return [(a, b, l - a - b) for a in range(l + 1) for b in range(l + 1 - a)]


def _solid_poly(l: int) -> np.ndarray:
    """Coefficients [2l+1, n_monomials] of R^l in the monomial basis.

    R^l is a homogeneous polynomial of degree l, so its coefficients follow
    exactly (up to rounding) from values at more points than monomials; they
    are fitted once by least squares over fixed random points.
    """
    if l not in _MONO_CACHE:
        mono = _monomials(l)
        pts = np.random.default_rng(4321 + l).standard_normal((4 * len(mono) + 8, 3))
        A = np.stack([pts[:, 0] ** a * pts[:, 1] ** b * pts[:, 2] ** c for a, b, c in mono], axis=1)
        coef, *_ = np.linalg.lstsq(A, solid_harmonics(l, pts), rcond=None)
        _MONO_CACHE[l] = coef.T
    return _MONO_CACHE[l]


def solid_harmonics_grad(l: int, r: np.ndarray) -> np.ndarray:
    """Gradient of the solid harmonics: [..., 2l+1, 3], d R^l_m / d r_a.

    The exact derivative of the monomial form of R^l (see _solid_poly).
    """
    r = np.asarray(r, dtype=np.float64)
    out = np.zeros(r.shape[:-1] + (2 * l + 1, 3))
    if l == 0:
        return out
    coef = _solid_poly(l)
    x, y, z = r[..., 0], r[..., 1], r[..., 2]
    pw = lambda v, e: v ** e if e > 0 else np.ones_like(v)
    for k, (a, b, c) in enumerate(_monomials(l)):
        if a:
            out[..., :, 0] += coef[:, k] * (a * pw(x, a - 1) * pw(y, b) * pw(z, c))[..., None]
        if b:
            out[..., :, 1] += coef[:, k] * (b * pw(x, a) * pw(y, b - 1) * pw(z, c))[..., None]
        if c:
            out[..., :, 2] += coef[:, k] * (c * pw(x, a) * pw(y, b) * pw(z, c - 1))[..., None]
    return out


# --------------------------------------------------------------------------
# Real coupling tensors
# --------------------------------------------------------------------------
@lru_cache(maxsize=None)
def real_cg(li: int, lf: int, lo: int) -> np.ndarray:
    """Real coupling tensor T[mo, mi, mf] of path (li, lf, lo), float64.

    T = sum U^{lo}[mo, muo] <li mui; lf muf | lo muo> conj(U^{li}[mi, mui])
    conj(U^{lf}[mf, muf]); real part for even li+lf+lo, imaginary part for odd.
    """
    Ui, Uf, Uo = real_basis(li), real_basis(lf), real_basis(lo)
    cg = np.zeros((2 * lo + 1, 2 * li + 1, 2 * lf + 1))
    for mui in range(-li, li + 1):
        for muf in range(-lf, lf + 1):
            muo = mui + muf
            if abs(muo) <= lo:
                cg[muo + lo, mui + li, muf + lf] = cg_complex(li, mui, lf, muf, lo, muo)
    T = np.einsum("ap,pqr,bq,cr->abc", Uo, cg, np.conj(Ui), np.conj(Uf))
    if (li + lf + lo) % 2 == 0:
        assert np.max(np.abs(T.imag)) < 1e-12
        return np.ascontiguousarray(T.real)
    assert np.max(np.abs(T.real)) < 1e-12
    return np.ascontiguousarray(T.imag)


def paths(lmax: int):
    """All (li, lf, lo) with |li-lf| <= lo <= li+lf and each <= lmax, in the
    order lo, then li, then lf ascending (the weight-row order)."""
    out = []
    for lo in range(lmax + 1):
        for li in range(lmax + 1):
            for lf in range(lmax + 1):
                if abs(li - lf) <= lo <= li + lf:
                    out.append((li, lf, lo))
    return out


# --------------------------------------------------------------------------
# Rotations
# --------------------------------------------------------------------------
def rot_z(a: float) -> np.ndarray:
    c, s = np.cos(a), np.sin(a)
    return np.array([[c, -s, 0.0], [s, c, 0.0], [0.0, 0.0, 1.0]])


def rot_y(a: float) -> np.ndarray:
    c, s = np.cos(a), np.sin(a)
    return np.array([[c, 0.0, s], [0.0, 1.0, 0.0], [-s, 0.0, c]])


def alignment_rotation(r: np.ndarray) -> np.ndarray:
    """Q in SO(3) with Q z^ = r^: Q = R_z(phi) R_y(theta); identity for r = 0.

    [EX] §2.1: "build the rotation that aligns the z axis with the position
    vector".
    """
    r = np.asarray(r, dtype=np.float64)
    n = np.linalg.norm(r)
    if n == 0.0:
        return np.eye(3)
    theta = np.arctan2(np.hypot(r[0], r[1]), r[2])     # accurate near both poles
    phi = np.arctan2(r[1], r[0])
    return rot_z(phi) @ rot_y(theta)


_FIT_DIRS = np.random.default_rng(12345).standard_normal((64, 3))


def wigner_D(l: int, Q: np.ndarray) -> np.ndarray:
    """Real Wigner-D matrix of degree l, defined by Y_l(Q u) = D Y_l(u).

    Solved by least squares over 64 fixed directions; exact up to rounding
    because the real harmonics of degree l span a (2l+1)-dimensional space
    that rotations map into itself.
    """
    if l == 0:
        return np.ones((1, 1))
    Y0 = sph_harm_real(l, _FIT_DIRS)                       # [n, 2l+1]
    Y1 = sph_harm_real(l, _FIT_DIRS @ np.asarray(Q).T)     # [n, 2l+1]
    # Y1[n, a] = sum_b D[a, b] Y0[n, b]  ->  Y0 @ D^T = Y1
    Dt, *_ = np.linalg.lstsq(Y0, Y1, rcond=None)
    return Dt.T
