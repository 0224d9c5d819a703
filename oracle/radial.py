"""Radial weights of the convolution: Bessel basis, polynomial envelope and
the radial MLP, with their VJP (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

FlashCart (arXiv 2610.06409) App. B: a radial envelope makes edge
contributions vanish smoothly at the cutoff, keeping the energy twice
differentiable in the positions; App. E: the radial weights vanish with their
first two derivatives at the cutoff.  e3j (arXiv 2609.35099) Table 3: the
MACE(a) model has 8 radial (Bessel) functions and a 5 Angstrom cutoff.

The pages print no formulas; the readings used here (MACE's usual ones):
  b_n(d) = sqrt(2 / rc) sin(n pi d / rc) / d,          n = 1 .. n_basis
  u(d)   = 1 - (p+1)(p+2)/2 x^p + p(p+2) x^(p+1) - p(p+1)/2 x^(p+2),
           x = d / rc clipped to [0, 1], p = 6   (u(0) = 1; u, u', u'' = 0 at rc)
  w(d)   = u(d) * (W3 silu(W2 silu(W1 b(d))))        reshaped to [P, C]
with no biases and silu(z) = z / (1 + exp(-z)).  The fused radial path of
the convolution produces w on the chip from these pieces; its backward needs
the VJP: the gradient of <gw, w> with respect to d (forces) and to W1..W3.

fp64 NumPy, written step by step.
"""
from __future__ import annotations

import numpy as np

P_ENV = 6


def bessel(d, rc: float, n_basis: int = 8) -> np.ndarray:
    d = np.asarray(d, dtype=np.float64)
    n = np.arange(1, n_basis + 1)
    safe = np.maximum(d, 1e-12)
    return np.sqrt(2.0 / rc) * np.sin(n[None, :] * np.pi * d[:, None] / rc) / safe[:, None]


def bessel_grad(d, rc: float, n_basis: int = 8) -> np.ndarray:
    """d b_n / d d, [E, n_basis]."""
    d = np.asarray(d, dtype=np.float64)
    n = np.arange(1, n_basis + 1)[None, :]
    safe = np.maximum(d, 1e-12)[:, None]
    k = n * np.pi / rc
    return np.sqrt(2.0 / rc) * (k * np.cos(k * safe) / safe - np.sin(k * safe) / safe ** 2)


def envelope(d, rc: float, p: int = P_ENV) -> np.ndarray:
    x = np.clip(np.asarray(d, dtype=np.float64) / rc, 0.0, 1.0)
    return 1.0 - (p + 1) * (p + 2) / 2 * x ** p + p * (p + 2) * x ** (p + 1) - p * (p + 1) / 2 * x ** (p + 2)


def envelope_grad(d, rc: float, p: int = P_ENV) -> np.ndarray:
    d = np.asarray(d, dtype=np.float64)
    x = np.clip(d / rc, 0.0, 1.0)
    g = (-(p + 1) * (p + 2) / 2 * p * x ** (p - 1) + p * (p + 2) * (p + 1) * x ** p -
         p * (p + 1) / 2 * (p + 2) * x ** (p + 1)) / rc
    return np.where(d < rc, g, 0.0)


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _silu_grad(z):
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def radial_weights(d, rc: float, params, P: int, C: int, p: int = P_ENV) -> np.ndarray:
    """w [E, P, C] (fp64) for edge lengths d."""
    W1, W2, W3 = (np.asarray(W, dtype=np.float64) for W in params)
    b = bessel(d, rc, W1.shape[0])
    z3 = _silu(_silu(b @ W1) @ W2) @ W3
    return (envelope(d, rc, p)[:, None] * z3).reshape(len(b), P, C)


def radial_weights_vjp(d, rc: float, params, gw, p: int = P_ENV):
    """(g_d [E], [g_W1, g_W2, g_W3]) of <gw, w(d; W)>."""
    W1, W2, W3 = (np.asarray(W, dtype=np.float64) for W in params)
    gw = np.asarray(gw, dtype=np.float64).reshape(len(d), -1)
    b = bessel(d, rc, W1.shape[0])
    z1 = b @ W1
    h1 = _silu(z1)
    z2 = h1 @ W2
    h2 = _silu(z2)
    z3 = h2 @ W3
    u = envelope(d, rc, p)
    g_z3 = u[:, None] * gw
    g_u = (gw * z3).sum(1)
    g_W3 = h2.T @ g_z3
    g_z2 = (g_z3 @ W3.T) * _silu_grad(z2)
    g_W2 = h1.T @ g_z2
    g_z1 = (g_z2 @ W2.T) * _silu_grad(z1)
    g_W1 = b.T @ g_z1
    g_b = g_z1 @ W1.T
    g_d = (g_b * bessel_grad(d, rc, W1.shape[0])).sum(1) + g_u * envelope_grad(d, rc, p)
    return g_d, [g_W1, g_W2, g_W3]


def conv_with_radial(prob, N: int, senders, receivers, r, x, rc: float, params, gy=None):
    """The convolution with its weights produced from the edge lengths by the
    radial MLP: y = conv(x, r, w(|r|)).  With gy, also the backward through
    both routes of r: dr = (dY/dr)^T gY + g_d(|r|) r / |r|, plus dx and the
    MLP weight gradients.  Returns y or (y, dx, dr, [g_W1, g_W2, g_W3])."""
    from . import conv as oconv
    r64 = np.asarray(r, dtype=np.float64)
    d = np.linalg.norm(r64, axis=1)
    w = radial_weights(d, rc, params, prob.P, prob.C)
    if gy is None:
        return oconv.forward_bruteforce(prob, N, senders, receivers, r, x, w)
    y = oconv.forward_bruteforce(prob, N, senders, receivers, r, x, w)
    dx, dw, dr_ang = oconv.backward_bruteforce(prob, N, senders, receivers, r, x, w, gy)
    g_d, g_W = radial_weights_vjp(d, rc, params, dw)
    safe = np.where(d > 0, d, 1.0)
    dr = dr_ang + (g_d / safe)[:, None] * r64 * (d > 0)[:, None]
    return y, dx, dr, g_W
