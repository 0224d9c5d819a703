"""Node-local channel-diagonal tensor product, forward and backward (oracle).

Test infrastructure only (see ``oracle/__init__.py``).

FlashCart (arXiv 2610.06409) §5 and App. B: the node-local ladder builds
higher-order correlations by repeated pairwise products at each atom; each
step couples same-index channels of two node features along the admissible
paths and either retains every path's output (a learned linear map mixes
paths and channels afterwards) or sums weighted paths ("path-reduced").
App. D: channel-diagonal products with path retention or summation.

For node features u [N][D_u][C] and v [N][D_v][C] (natural-parity prefixes;
v plays the role the harmonics play in the convolution, so paths are
enumerated exactly as there with L_sh = L_v) and per-path, per-channel
weights w [P][C] (all ones for pure retention):

    y[i, o3(p) + m3, c] = sum_p w[p, c] sum_{m1, m2} C_p[m1, m2, m3] u[i, l1 m1, c] v[i, l2 m2, c]

with o3(p) the summed layout (paths sharing an output irrep add) or the
per-path layout of ``Problem(per_path=True)``.  Backward given gy:

    du[i, l1 m1, c] = sum_p w[p, c] sum_{m2, m3} C_p v[i, l2 m2, c] gy[i, o3(p) + m3, c]
    dv[i, l2 m2, c] = sum_p w[p, c] sum_{m1, m3} C_p u[i, l1 m1, c] gy[i, o3(p) + m3, c]
    dw[p, c]        = sum_i sum_{m1, m2, m3} C_p u v gy

NumPy einsum, fp64.
"""
from __future__ import annotations

import numpy as np

from .conv import Problem


def _f64(t):
    return np.asarray(t, dtype=np.float64)


def node_product(prob: Problem, u, v, w=None) -> np.ndarray:
    u, v = _f64(u), _f64(v)
    N = u.shape[0]
    w = np.ones((prob.P, prob.C)) if w is None else _f64(w)
    y = np.zeros((N, prob.D_out, prob.C))
    for p, q in enumerate(prob.paths):
        d1, d2, d3 = 2 * q["l1"] + 1, 2 * q["l2"] + 1, 2 * q["l3"] + 1
        ub = u[:, q["off1"]:q["off1"] + d1, :]
        vb = v[:, q["off2"]:q["off2"] + d2, :]
        y[:, q["off3"]:q["off3"] + d3, :] += w[p] * np.einsum("abk,nac,nbc->nkc", prob.cg(p), ub, vb)
    return y


def node_product_backward(prob: Problem, u, v, w, gy):
    """(du, dv, dw); w None means all ones (dw is still returned)."""
    u, v, gy = _f64(u), _f64(v), _f64(gy)
    w = np.ones((prob.P, prob.C)) if w is None else _f64(w)
    du, dv = np.zeros_like(u), np.zeros_like(v)
    dw = np.zeros((prob.P, prob.C))
    for p, q in enumerate(prob.paths):
        d1, d2, d3 = 2 * q["l1"] + 1, 2 * q["l2"] + 1, 2 * q["l3"] + 1
        Cp = prob.cg(p)
        ub = u[:, q["off1"]:q["off1"] + d1, :]
        vb = v[:, q["off2"]:q["off2"] + d2, :]
        gb = gy[:, q["off3"]:q["off3"] + d3, :]
        du[:, q["off1"]:q["off1"] + d1, :] += w[p] * np.einsum("abk,nbc,nkc->nac", Cp, vb, gb)
        dv[:, q["off2"]:q["off2"] + d2, :] += w[p] * np.einsum("abk,nac,nkc->nbc", Cp, ub, gb)
        dw[p] = np.einsum("abk,nac,nbc,nkc->c", Cp, ub, vb, gb)
    return du, dv, dw
