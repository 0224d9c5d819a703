"""Pins for the oracle's real spherical harmonics and their gradient (no GPU).

FlashCart (arXiv 2610.06409), §2 and App. B: the degree-l direction tensors
are the real spherical tensors of the edge direction; forces need their
gradient.  The convention (component normalisation, z polar, cos for m>0 and
sin for m<0, positive leading coefficients) is pinned by closed forms,
quadrature orthonormality, the addition theorem (SciPy's Legendre), and finite
differences.
"""
import numpy as np
import pytest
from scipy.special import eval_legendre

from oracle.sh import sh, sh_grad

s3, s5, s7, s15, s105 = (np.sqrt(v) for v in (3.0, 5.0, 7.0, 15.0, 105.0))


def closed_forms(u):
    """Component-normalised real harmonics l <= 3 written out as Cartesian
    polynomials of the unit vector (textbook forms times sqrt(4 pi))."""
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    a3 = np.sqrt(35.0 / 2.0) / 2.0
    a1 = np.sqrt(21.0 / 2.0) / 2.0
    cols = [
        np.ones_like(x),
        s3 * y, s3 * z, s3 * x,
        s15 * x * y, s15 * y * z, s5 / 2 * (3 * z * z - 1), s15 * x * z, s15 / 2 * (x * x - y * y),
        a3 * (3 * x * x - y * y) * y, s105 * x * y * z, a1 * y * (5 * z * z - 1),
        s7 / 2 * (5 * z ** 3 - 3 * z), a1 * x * (5 * z * z - 1), s105 / 2 * (x * x - y * y) * z,
        a3 * (x * x - 3 * y * y) * x,
    ]
    return np.stack(cols, axis=1)


def rand_unit(n, seed):
    v = np.random.default_rng(seed).standard_normal((n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def test_closed_forms_l3():
    u = rand_unit(200, 1)
    assert np.max(np.abs(sh(u, 3) - closed_forms(u))) < 1e-12


def test_scale_invariance():
    u = rand_unit(50, 2)
    assert np.max(np.abs(sh(3.7 * u, 3) - sh(u, 3))) < 1e-12


@pytest.mark.parametrize("L", [3, 5])
def test_component_normalisation(L):
    Y = sh(rand_unit(100, 3), L)
    for l in range(L + 1):
        assert np.max(np.abs((Y[:, l * l:(l + 1) ** 2] ** 2).sum(1) - (2 * l + 1))) < 1e-11


def test_quadrature_orthonormality():
    """int Y_lm Y_l'm' dOmega / 4pi = delta (Gauss-Legendre in cos(theta) x
    uniform phi, exact for the degree-2L integrand)."""
    L = 4
    zs, wz = np.polynomial.legendre.leggauss(L + 2)
    nphi = 2 * L + 3
    phi = 2 * np.pi * np.arange(nphi) / nphi
    Z, PHI = np.meshgrid(zs, phi, indexing="ij")
    rho = np.sqrt(1 - Z ** 2)
    u = np.stack([rho * np.cos(PHI), rho * np.sin(PHI), Z], -1).reshape(-1, 3)
    wts = (wz[:, None] * np.ones(nphi)[None, :] / nphi / 2.0).reshape(-1)
    Y = sh(u, L)
    G = np.einsum("q,qa,qb->ab", wts, Y, Y)
    assert np.max(np.abs(G - np.eye((L + 1) ** 2))) < 1e-12


def test_addition_theorem():
    u, v = rand_unit(100, 4), rand_unit(100, 5)
    Yu, Yv = sh(u, 4), sh(v, 4)
    c = (u * v).sum(1)
    for l in range(5):
        lhs = (Yu[:, l * l:(l + 1) ** 2] * Yv[:, l * l:(l + 1) ** 2]).sum(1)
        assert np.max(np.abs(lhs - (2 * l + 1) * eval_legendre(l, c))) < 1e-11


def test_parity():
    u = rand_unit(40, 6)
    Yp, Ym = sh(u, 3), sh(-u, 3)
    for l in range(4):
        sl = slice(l * l, (l + 1) ** 2)
        assert np.max(np.abs(Ym[:, sl] - (-1) ** l * Yp[:, sl])) < 1e-12


def test_gradient_finite_differences():
    rng = np.random.default_rng(9)
    r = rng.standard_normal((60, 3)) * 2.0
    g = sh_grad(r, 3)
    h = 1e-6
    for j in range(3):
        dr = np.zeros(3)
        dr[j] = h
        fd = (sh(r + dr, 3) - sh(r - dr, 3)) / (2 * h)
        assert np.max(np.abs(fd - g[:, :, j])) < 1e-7 * max(1.0, np.max(np.abs(g)))


def test_gradient_is_tangential_and_scales():
    rng = np.random.default_rng(10)
    r = rng.standard_normal((30, 3))
    g = sh_grad(r, 3)
    assert np.max(np.abs(np.einsum("ekj,ej->ek", g, r))) < 1e-12
    # Y(r/|r|) is homogeneous of degree 0, so grad scales as 1/|r|
    assert np.max(np.abs(sh_grad(2.5 * r, 3) * 2.5 - g)) < 1e-12


def test_zero_length_rule():
    r = np.array([[0.0, 0.0, 0.0], [1e-13, 0.0, 0.0]])
    Y = sh(r, 3)
    assert np.all(Y[:, 0] == 1.0) and np.all(Y[:, 1:] == 0.0)
    assert np.all(sh_grad(r, 3) == 0.0)
