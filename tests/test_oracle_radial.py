"""Pins for the oracle's radial weights (no GPU): Bessel basis, polynomial
envelope, radial MLP and its VJP.

FlashCart (arXiv 2610.06409) App. B and App. E: the radial weights vanish
with their first two derivatives at the cutoff; e3j (arXiv 2609.35099)
Table 3: 8 radial functions, 5 Angstrom cutoff.  What pins the oracle:
* the envelope as a polynomial built by numpy.polynomial (a library route):
  1 at 0, and value, first and second derivative 0 at the cutoff;
* Bessel orthonormality: integral_0^rc b_n b_m d^2 dd = delta_nm
  (Gauss-Legendre quadrature);
* the MLP and the VJP against torch (matmul, SiLU, autograd) in fp64;
* the VJP in d against central differences;
* the seeded water-box generator gives the oracle's weights (fp32).
"""
import numpy as np
import torch
from numpy.polynomial import Polynomial

from equivariant_gnn_message_edge_b200 import workloads as wl
from oracle import radial as R

RC = 5.0


def test_envelope_is_c2_at_the_cutoff():
    p = R.P_ENV
    poly = Polynomial.basis(0) - (p + 1) * (p + 2) / 2 * Polynomial.basis(p) + p * (p + 2) * Polynomial.basis(p + 1) \
        - p * (p + 1) / 2 * Polynomial.basis(p + 2)
    assert abs(poly(0.0) - 1.0) < 1e-15
    for k in range(3):
        assert abs(poly.deriv(k)(1.0)) < 1e-12
    x = np.linspace(0, 1, 11)
    assert np.max(np.abs(R.envelope(x * RC, RC) - poly(x))) < 1e-14
    assert np.max(np.abs(R.envelope_grad(x[:-1] * RC, RC) - poly.deriv(1)(x[:-1]) / RC)) < 1e-12
    assert np.all(R.envelope(np.array([RC, 6.0, 9.0]), RC) == 0.0)
    assert np.all(R.envelope_grad(np.array([RC, 6.0]), RC) == 0.0)


def test_bessel_basis_is_orthonormal_with_weight_d2():
    xg, wg = np.polynomial.legendre.leggauss(200)
    d = 0.5 * RC * (xg + 1.0)
    b = R.bessel(d, RC, 8)
    G = np.einsum("q,qn,qm->nm", 0.5 * RC * wg * d ** 2, b, b)
    assert np.max(np.abs(G - np.eye(8))) < 1e-12


def _params(P, C, seed=0):
    rng = np.random.default_rng(seed)
    dims = [8, 16, 16, P * C]
    return [rng.standard_normal((a, b)) / np.sqrt(a) for a, b in zip(dims[:-1], dims[1:])]


def test_mlp_and_vjp_match_torch_autograd():
    P, C = 3, 4
    params = _params(P, C)
    rng = np.random.default_rng(1)
    d = rng.uniform(0.3, 6.0, 50)                       # some beyond the cutoff
    gw = rng.standard_normal((50, P, C))
    dt = torch.tensor(d, dtype=torch.float64, requires_grad=True)
    Wt = [torch.tensor(W, requires_grad=True) for W in params]
    n = torch.arange(1, 9, dtype=torch.float64)
    b = (2.0 / RC) ** 0.5 * torch.sin(n * torch.pi * dt[:, None] / RC) / dt[:, None]
    x = torch.clamp(dt / RC, 0.0, 1.0)
    p = R.P_ENV
    u = 1 - (p + 1) * (p + 2) / 2 * x ** p + p * (p + 2) * x ** (p + 1) - p * (p + 1) / 2 * x ** (p + 2)
    z = torch.nn.functional.silu(torch.nn.functional.silu(b @ Wt[0]) @ Wt[1]) @ Wt[2]
    w = (u[:, None] * z).reshape(50, P, C)
    assert np.max(np.abs(R.radial_weights(d, RC, params, P, C) - w.detach().numpy())) < 1e-12
    (w * torch.tensor(gw)).sum().backward()
    g_d, g_W = R.radial_weights_vjp(d, RC, params, gw)
    assert np.max(np.abs(g_d - dt.grad.numpy())) < 1e-10 * max(1.0, np.max(np.abs(g_d)))
    for a, t in zip(g_W, Wt):
        assert np.max(np.abs(a - t.grad.numpy())) < 1e-10 * max(1.0, np.max(np.abs(a)))


def test_vjp_in_d_matches_central_differences():
    P, C = 2, 3
    params = _params(P, C, seed=4)
    rng = np.random.default_rng(5)
    d = rng.uniform(0.5, 4.9, 20)
    gw = rng.standard_normal((20, P, C))
    g_d, _ = R.radial_weights_vjp(d, RC, params, gw)
    h = 1e-6
    fd = ((R.radial_weights(d + h, RC, params, P, C) - R.radial_weights(d - h, RC, params, P, C)) * gw).sum((1, 2)) / (2 * h)
    assert np.max(np.abs(fd - g_d)) < 1e-6 * max(1.0, np.max(np.abs(g_d)))


def test_water_box_generator_matches_the_oracle():
    P, C = 5, 8
    params = wl.radial_mlp_params(P, C, hidden=16, n_bessel=8, seed=3)
    rng = np.random.default_rng(6)
    r = (rng.standard_normal((40, 3)) * 2).astype(np.float32)
    dummy = np.zeros(40, bool)
    dummy[::7] = True
    w = wl.radial_weights(r, RC, params, P, C, is_dummy=dummy)
    ref = R.radial_weights(np.linalg.norm(r.astype(np.float64), axis=1), RC, params, P, C)
    ref[dummy] = 0.0
    assert np.max(np.abs(w - ref)) < 1e-5 * np.max(np.abs(ref)) + 1e-6
    assert np.all(w[dummy] == 0.0)


def test_conv_with_radial_weights_backward_matches_differences():
    """The fused path's oracle: y = conv(x, r, w(|r|)); the gradient of
    <gy, y> in r has an angular part (harmonics) and a radial part (the MLP),
    and in the MLP weights; central differences of the composition check
    both routes (everything fp64)."""
    from oracle.conv import Problem
    prob = Problem("0e+1o+2e", 2, "0e+1o+2e", 3)
    rng = np.random.default_rng(9)
    N, E = 6, 20
    s = rng.integers(0, N, E).astype(np.int32)
    rcv = rng.integers(0, N, E).astype(np.int32)
    r = rng.standard_normal((E, 3)) * 1.5
    x = rng.standard_normal((N, prob.D_in, 3))
    gy = rng.standard_normal((N, prob.D_out, 3))
    params = _params(prob.P, prob.C, seed=10)
    y, dx, dr, g_W = R.conv_with_radial(prob, N, s, rcv, r, x, RC, params, gy)

    def S(rr, pp):
        return float((gy * R.conv_with_radial(prob, N, s, rcv, rr, x, RC, pp)).sum())
    h = 1e-5
    dirn = rng.standard_normal(r.shape)
    fd = (S(r + h * dirn, params) - S(r - h * dirn, params)) / (2 * h)
    assert abs(fd - (dr * dirn).sum()) < 1e-4 * max(1.0, abs(fd))
    for k in range(3):
        dW = rng.standard_normal(params[k].shape)
        pp = [W.copy() for W in params]
        pm = [W.copy() for W in params]
        pp[k] += h * dW
        pm[k] -= h * dW
        fd = (S(r, pp) - S(r, pm)) / (2 * h)
        assert abs(fd - (g_W[k] * dW).sum()) < 1e-4 * max(1.0, abs(fd))
