"""Pins for the oracle's double backward and its SH Hessian (no GPU).

FlashCart (arXiv 2610.06409) §2 (training on forces differentiates the force
evaluation), §3 and App. C (VJP-of-VJP of weighted bilinear products).

The double backward is the gradient of S = <a, dx> + <b, dw> + <q, dr>, with
(dx, dw, dr) the first-order backward, which the other oracle tests pin.  So:
* directional central differences of S (fp64, through the first-order
  NumPy brute force) must match <grad, direction> for x, w, gy and r;
* S is linear in gy, so <dS/dgy, gy> = S; dx and dr are linear in w and dw
  does not depend on w, so <dS/dw, w> = <a, dx> + <q, dr>; likewise
  <dS/dx, x> = <b, dw> + <q, dr>; dx and dw depend on r only through the
  direction (degree 0) and dr is homogeneous of degree -1, so
  <dS/dr, r> = -<q, dr>  (Euler's theorem, exact).
The Hessian of the harmonics is built from homogeneous polynomials, not
from the gradient code, and is pinned by central differences of the
gradient, symmetry, and Euler's identity H r = -dY/dr (Y has degree 0).
"""
import numpy as np
import pytest

from oracle import conv
from oracle.dbl import double_backward_bruteforce
from oracle.sh import sh_grad, sh_hessian
from tests.helpers import small_problem

CASES = [dict(L_in=1, L_sh=2, L_out=2), dict(L_in=2, L_sh=2, L_out=2), dict(L_in=3, L_sh=3, L_out=3),
         dict(L_in=2, L_sh=1, L_out=3), dict(L_in=1, L_sh=0, L_out=1)]


@pytest.mark.parametrize("L", [0, 1, 2, 3])
def test_sh_hessian_pins(L):
    rng = np.random.default_rng(L)
    r = rng.standard_normal((40, 3)) * rng.uniform(0.3, 3.0, (40, 1))
    H = sh_hessian(r, L)
    J = sh_grad(r, L)
    h = 1e-5
    fd = np.zeros_like(H)
    for k in range(3):
        e = np.zeros(3)
        e[k] = h
        fd[..., :, k] = (sh_grad(r + e, L) - sh_grad(r - e, L)) / (2 * h)
    scale = max(1.0, np.max(np.abs(H)))
    assert np.max(np.abs(H - fd)) < 1e-7 * scale
    assert np.max(np.abs(H - np.swapaxes(H, -1, -2))) < 1e-12 * scale
    assert np.max(np.abs(np.einsum("ekij,ej->eki", H, r) + J)) < 1e-12 * scale
    assert np.all(sh_hessian(np.zeros((2, 3)), L) == 0.0)


def _setup(case, seed, N=8, E=30, C=3):
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=E, C=C, seed=seed, **case)
    rng = np.random.default_rng(seed + 100)
    a = rng.standard_normal(x.shape)
    b = rng.standard_normal(w.shape)
    q = rng.standard_normal(r.shape)
    f = lambda t: np.asarray(t, dtype=np.float64)
    return prob, s, rcv, f(r), f(x), f(w), f(gy), a, b, q


def _S(prob, N, s, rcv, r, x, w, gy, a, b, q):
    dx, dw, dr = conv.backward_bruteforce(prob, N, s, rcv, r, x, w, gy)
    return float((a * dx).sum() + (b * dw).sum() + (q * dr).sum()), (dx, dw, dr)


@pytest.mark.parametrize("case", CASES)
def test_double_backward_matches_central_differences(case):
    N = 8
    prob, s, rcv, r, x, w, gy, a, b, q = _setup(case, seed=3)
    g_x, g_w, g_gy, g_r = double_backward_bruteforce(prob, N, s, rcv, r, x, w, gy, a, b, q)
    rng = np.random.default_rng(11)
    h = 1e-6
    args = dict(r=r, x=x, w=w, gy=gy)
    for name, g in (("x", g_x), ("w", g_w), ("gy", g_gy), ("r", g_r)):
        d = rng.standard_normal(args[name].shape)
        plus, minus = dict(args), dict(args)
        plus[name] = args[name] + h * d
        minus[name] = args[name] - h * d
        Sp, _ = _S(prob, N, s, rcv, plus["r"], plus["x"], plus["w"], plus["gy"], a, b, q)
        Sm, _ = _S(prob, N, s, rcv, minus["r"], minus["x"], minus["w"], minus["gy"], a, b, q)
        fd = (Sp - Sm) / (2 * h)
        an = float((g * d).sum())
        assert abs(fd - an) < 1e-6 * max(1.0, abs(an)), (name, fd, an)


@pytest.mark.parametrize("case", CASES)
def test_double_backward_euler_identities(case):
    N = 8
    prob, s, rcv, r, x, w, gy, a, b, q = _setup(case, seed=5)
    g_x, g_w, g_gy, g_r = double_backward_bruteforce(prob, N, s, rcv, r, x, w, gy, a, b, q)
    S, (dx, dw, dr) = _S(prob, N, s, rcv, r, x, w, gy, a, b, q)
    A, Bt, Q = (a * dx).sum(), (b * dw).sum(), (q * dr).sum()
    tol = 1e-11 * max(1.0, abs(A) + abs(Bt) + abs(Q))
    assert abs((g_gy * gy).sum() - S) < tol
    assert abs((g_w * w).sum() - (A + Q)) < tol
    assert abs((g_x * x).sum() - (Bt + Q)) < tol
    assert abs((g_r * r).sum() + Q) < tol


def test_double_backward_zero_cotangents_give_zero():
    prob, s, rcv, r, x, w, gy, a, b, q = _setup(CASES[1], seed=7)
    z = double_backward_bruteforce(prob, 8, s, rcv, r, x, w, gy, 0 * a, 0 * b, 0 * q)
    assert all(np.all(t == 0.0) for t in z)


def test_double_backward_zero_length_edges():
    """A zero-length edge has Y_0 = 1, Y_l>0 = 0 and no r-dependence: its
    rho and its dS/dr vanish."""
    prob, s, rcv, r, x, w, gy, a, b, q = _setup(CASES[1], seed=9)
    r[0] = 0.0
    g_x, g_w, g_gy, g_r = double_backward_bruteforce(prob, 8, s, rcv, r, x, w, gy, a, b, q)
    assert np.all(g_r[0] == 0.0)
    assert np.all(np.isfinite(g_x)) and np.all(np.isfinite(g_gy)) and np.all(np.isfinite(g_w))
