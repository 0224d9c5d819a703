"""Real spherical harmonics of the edge direction and their gradient
(oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

FlashCart (arXiv 2610.06409), §2 and App. B: the degree-l direction tensors
are the degree-l real spherical tensors of the unit edge direction; forces are
gradients of the energy (§2), which needs dY/dr.  The pages fix no
normalisation or phase; the reading used here (MACE's usual one):

* z is the polar axis, m = -l..l; Y_{l,m>0} ~ cos(m phi), Y_{l,m<0} ~ sin(|m| phi),
  positive leading coefficients (no Condon-Shortley phase in the real basis);
* component normalisation: sum_m Y_lm(u)^2 = 2l+1 for every unit u.

Construction (textbook): with Q_l^m(z) = d^m P_l / dz^m (Legendre P_l) and
(x + i y)^m = C_m + i S_m,
    Y_lm = N_lm Q_l^|m|(z) * (C_|m| if m >= 0 else S_|m|),
    N_lm = sqrt((2l+1) (2 - delta_m0) (l-|m|)! / (l+|m|)!).
The expression is a polynomial f(x, y, z) that equals Y on the unit sphere, so
for an edge vector r with u = r/|r|:
    dY/dr = (I - u u^T) grad f(u) / |r|.
Zero-length edges (|r| < 1e-12): u = 0, Y_0 = 1, Y_{l>0} = 0, dY/dr = 0.
"""
from __future__ import annotations

from math import factorial

import numpy as np
from numpy.polynomial import legendre as npleg
from numpy.polynomial import polynomial as nppoly

ZERO_LEN = 1e-12


def _legendre_power_coeffs(l: int) -> np.ndarray:
    c = np.zeros(l + 1)
    c[l] = 1.0
    return npleg.leg2poly(c)


def _norm(l: int, am: int) -> float:
    return np.sqrt((2 * l + 1) * (1 if am == 0 else 2) * factorial(l - am) / factorial(l + am))


def _unit(r: np.ndarray):
    r = np.asarray(r, dtype=np.float64)
    n = np.linalg.norm(r, axis=-1)
    zero = n < ZERO_LEN
    safe = np.where(zero, 1.0, n)
    u = r / safe[..., None]
    u[zero] = 0.0
    return u, n, zero


def sh(r: np.ndarray, L: int) -> np.ndarray:
    """Y[..., l*l + m + l] for l = 0..L of the directions of r (fp64)."""
    u, _, zero = _unit(r)
    x, y, z = u[..., 0], u[..., 1], u[..., 2]
    out = np.zeros(u.shape[:-1] + ((L + 1) ** 2,))
    xy = x + 1j * y
    for l in range(L + 1):
        P = _legendre_power_coeffs(l)
        for m in range(-l, l + 1):
            am = abs(m)
            Q = nppoly.polyval(z, nppoly.polyder(P, am)) if am <= l else 0.0
            cs = xy ** am
            ang = cs.real if m >= 0 else cs.imag
            out[..., l * l + m + l] = _norm(l, am) * Q * ang
    out[zero] = 0.0
    out[zero, 0] = 1.0
    return out


def sh_grad(r: np.ndarray, L: int) -> np.ndarray:
    """dY/dr, shape [..., (L+1)^2, 3] (fp64)."""
    u, n, zero = _unit(r)
    x, y, z = u[..., 0], u[..., 1], u[..., 2]
    xy = x + 1j * y
    g = np.zeros(u.shape[:-1] + ((L + 1) ** 2, 3))
    for l in range(L + 1):
        P = _legendre_power_coeffs(l)
        for m in range(-l, l + 1):
            am = abs(m)
            Qp = nppoly.polyder(P, am)
            Q = nppoly.polyval(z, Qp)
            dQ = nppoly.polyval(z, nppoly.polyder(Qp, 1)) if len(Qp) > 1 else np.zeros_like(z)
            cs = xy ** am
            # d/dx (x+iy)^a = a (x+iy)^(a-1);  d/dy (x+iy)^a = i a (x+iy)^(a-1)
            d = am * xy ** (am - 1) if am > 0 else np.zeros_like(xy)
            if m >= 0:
                ang, dax, day = cs.real, d.real, (1j * d).real
            else:
                ang, dax, day = cs.imag, d.imag, (1j * d).imag
            N = _norm(l, am)
            k = l * l + m + l
            g[..., k, 0] = N * Q * dax
            g[..., k, 1] = N * Q * day
            g[..., k, 2] = N * dQ * ang
    # project out the radial part and divide by |r|
    radial = np.einsum("...kj,...j->...k", g, u)
    g = g - radial[..., None] * u[..., None, :]
    safe = np.where(zero, 1.0, n)
    g = g / safe[..., None, None]
    g[zero] = 0.0
    return g
