"""Double backward (VJP of the backward) of the convolution (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

FlashCart (arXiv 2610.06409) §2: training on forces needs the derivative of
the force evaluation; §3 and App. C: for a weighted bilinear product the
VJP-of-VJP follows from bilinearity and reduces to linear-map evaluations;
App. D: the VJP-of-VJP sums receiver contributions to the derivative of the
incoming gradient.

With the forward written as the multilinear form
    F(x, w, Y, gy) = <gy, y> = sum_e sum_p sum_c w[e,p,c] sum C_p x[s,l1,m1,c] Y[e,l2,m2] gy[i,l3,m3,c],
the backward outputs are dx = dF/dx, dw = dF/dw and dr = J(r)^T gY with
gY = dF/dY and J = dY/dr.  Given cotangents a (of dx), b (of dw) and q (of
dr), the double backward returns the gradient of
    S = <a, dx> + <b, dw> + <q, dr>
with respect to x, w, gy and r.  Because F is linear in each argument,
    <a, dx> = F(a, w, Y, gy),  <b, dw> = F(x, b, Y, gy),  <q, dr> = F(x, w, rho, gy)
with rho[e] = J(r_e) q[e], so
    dS/dgy = y(a, w, Y) + y(x, b, Y) + y(x, w, rho)                 (receiver sums)
    dS/dx  = dx(b, Y, gy) + dx(w, rho, gy)                          (sender sums)
    dS/dw  = dw(a, Y, gy) + dw(x, rho, gy)                          (per edge)
    dS/dr  = J^T [gY(a, w, gy) + gY(x, b, gy)] + H(r; gY(x, w, gy)) q
where y(.), dx(.), dw(.), gY(.) are the first-order formulas with the named
arguments substituted and H(r; g) = d^2/dr^2 sum_k g_k Y_k(r).

``double_backward_bruteforce`` materialises per-edge terms in NumPy (fp64);
small inputs only.
"""
from __future__ import annotations

import numpy as np

from .conv import Problem
from .sh import sh, sh_grad, sh_hessian


def double_backward_bruteforce(prob: Problem, N: int, senders, receivers, r, x, w, gy, a, b, q):
    """(g_x [N,D_in,C], g_w [E,P,C], g_gy [N,D_out,C], g_r [E,3]), fp64."""
    senders = np.asarray(senders)
    receivers = np.asarray(receivers)
    r = np.asarray(r, dtype=np.float64)
    f = lambda t: np.asarray(t, dtype=np.float64)
    x, w, gy, a, b, q = f(x), f(w), f(gy), f(a), f(b), f(q)
    L = prob.L_sh
    Y = sh(r, L)
    J = sh_grad(r, L)                                   # [E, D_sh, 3]
    rho = np.einsum("ekj,ej->ek", J, q)                 # J q
    E = len(senders)
    xs, as_, gyr = x[senders], a[senders], gy[receivers]
    g_gy_e = np.zeros((E, prob.D_out, prob.C))
    g_x_e = np.zeros((E, prob.D_in, prob.C))
    g_w = np.zeros((E, prob.P, prob.C))
    gYv = np.zeros((E, prob.D_sh))                      # gY(a, w, gy) + gY(x, b, gy)
    gY1 = np.zeros((E, prob.D_sh))                      # gY(x, w, gy)
    for p, pq in enumerate(prob.paths):
        d1, d2, d3 = 2 * pq["l1"] + 1, 2 * pq["l2"] + 1, 2 * pq["l3"] + 1
        o1, o2, o3 = pq["off1"], pq["off2"], pq["off3"]
        Cp = prob.cg(p)
        xb, ab = xs[:, o1:o1 + d1, :], as_[:, o1:o1 + d1, :]
        gb = gyr[:, o3:o3 + d3, :]
        Yb, Rb = Y[:, o2:o2 + d2], rho[:, o2:o2 + d2]
        wp, bp = w[:, p, None, :], b[:, p, None, :]
        msg = lambda yv, xv: np.einsum("abk,eb,eac->ekc", Cp, yv, xv)
        g_gy_e[:, o3:o3 + d3, :] += wp * msg(Yb, ab) + bp * msg(Yb, xb) + wp * msg(Rb, xb)
        uY = np.einsum("abk,eb,ekc->eac", Cp, Yb, gb)
        uR = np.einsum("abk,eb,ekc->eac", Cp, Rb, gb)
        g_x_e[:, o1:o1 + d1, :] += bp * uY + wp * uR
        g_w[:, p, :] = np.einsum("eac,eac->ec", ab, uY) + np.einsum("eac,eac->ec", xb, uR)
        Ga = np.einsum("abk,eac,ekc->ebc", Cp, ab, gb)
        Gx = np.einsum("abk,eac,ekc->ebc", Cp, xb, gb)
        gYv[:, o2:o2 + d2] += np.einsum("ebc,ec->eb", Ga, w[:, p]) + np.einsum("ebc,ec->eb", Gx, b[:, p])
        gY1[:, o2:o2 + d2] += np.einsum("ebc,ec->eb", Gx, w[:, p])
    g_gy = np.zeros((N, prob.D_out, prob.C))
    np.add.at(g_gy, receivers, g_gy_e)
    g_x = np.zeros((N, prob.D_in, prob.C))
    np.add.at(g_x, senders, g_x_e)
    H = sh_hessian(r, L)
    g_r = np.einsum("ekj,ek->ej", J, gYv) + np.einsum("ekij,ek,ej->ei", H, gY1, q)
    return g_x, g_w, g_gy, g_r
