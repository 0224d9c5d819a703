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


# --------------------------------------------------------------------------
# Second derivatives (double backward of the convolution)
# --------------------------------------------------------------------------
# An independent construction: Y_lm(r) = P_lm(r) / |r|^l with P_lm the
# homogeneous degree-l polynomial that equals Y_lm on the unit sphere,
#     P_lm = N_lm sum_k q_k z^k (x^2+y^2+z^2)^((l-|m|-k)/2) A_m(x, y),
# q_k the coefficients of d^|m| P_l / dz^|m| (only k = l-|m| mod 2 occur) and
# A_m = Re or Im of (x + i y)^|m|.  Polynomials are dicts {(i, j, k): c}.

def _pmul(p, q):
    out = {}
    for (a, b, c), u in p.items():
        for (d, e, f), v in q.items():
            key = (a + d, b + e, c + f)
            out[key] = out.get(key, 0.0) + u * v
    return out


def _padd(p, q, s=1.0):
    out = dict(p)
    for k, v in q.items():
        out[k] = out.get(k, 0.0) + s * v
    return out


def _pderiv(p, var):
    out = {}
    for key, c in p.items():
        if key[var] == 0:
            continue
        k2 = list(key)
        k2[var] -= 1
        out[tuple(k2)] = out.get(tuple(k2), 0.0) + c * key[var]
    return out


def _peval(p, r):
    x, y, z = r[..., 0], r[..., 1], r[..., 2]
    out = np.zeros(r.shape[:-1])
    for (a, b, c), v in p.items():
        out = out + v * x ** a * y ** b * z ** c
    return out


def _homogeneous(l: int, m: int) -> dict:
    am = abs(m)
    Q = nppoly.polyder(_legendre_power_coeffs(l), am) if am <= l else np.zeros(1)
    rho2 = {(2, 0, 0): 1.0, (0, 2, 0): 1.0, (0, 0, 2): 1.0}
    # (x + i y)^am expanded: sum_j binom(am, j) x^(am-j) (i y)^j
    from math import comb
    A = {}
    for j in range(am + 1):
        ij = 1j ** j
        part = ij.real if m >= 0 else ij.imag
        if abs(part) > 0:
            A[(am - j, j, 0)] = A.get((am - j, j, 0), 0.0) + comb(am, j) * part
    P = {}
    for k, qk in enumerate(Q):
        if qk == 0.0:
            continue
        e = l - am - k
        assert e % 2 == 0 and e >= 0
        term = {(0, 0, k): qk}
        for _ in range(e // 2):
            term = _pmul(term, rho2)
        P = _padd(P, term)
    P = _pmul(P, A) if A else {}
    return {key: _norm(l, am) * v for key, v in P.items()}


def sh_hessian(r: np.ndarray, L: int) -> np.ndarray:
    """d^2 Y / dr dr^T, shape [..., (L+1)^2, 3, 3] (fp64); zero-length edges
    give 0.  Built from the homogeneous polynomials above (quotient rule on
    P / |r|^l), not from ``sh_grad``."""
    r = np.asarray(r, dtype=np.float64)
    n = np.linalg.norm(r, axis=-1)
    zero = n < ZERO_LEN
    rs = np.where(zero[..., None], 1.0, r)
    ns = np.where(zero, 1.0, n)
    H = np.zeros(r.shape[:-1] + ((L + 1) ** 2, 3, 3))
    eye = np.eye(3)
    for l in range(1, L + 1):
        s = ns ** (-l)
        ds = -l * ns[..., None] ** (-l - 2) * rs                                    # grad |r|^-l
        hs = (-l * ns[..., None, None] ** (-l - 2) * eye +
              l * (l + 2) * ns[..., None, None] ** (-l - 4) * rs[..., :, None] * rs[..., None, :])
        for m in range(-l, l + 1):
            P = _homogeneous(l, m)
            g = [_pderiv(P, a) for a in range(3)]
            Pv = _peval(P, rs)
            gv = np.stack([_peval(g[a], rs) for a in range(3)], axis=-1)
            hv = np.stack([np.stack([_peval(_pderiv(g[a], b), rs) for b in range(3)], axis=-1)
                           for a in range(3)], axis=-2)
            k = l * l + m + l
            H[..., k, :, :] = (s[..., None, None] * hv + gv[..., :, None] * ds[..., None, :] +
                               ds[..., :, None] * gv[..., None, :] + Pv[..., None, None] * hs)
    H[zero] = 0.0
    return H
