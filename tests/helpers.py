"""Shared test helpers: small problems, Wigner matrices, tolerance check."""
from __future__ import annotations

import numpy as np

from oracle.irreps import block_offsets, parse_irreps
from oracle.sh import sh


def wigner_real(R: np.ndarray, l: int, n_pts: int = 64, seed: int = 0) -> np.ndarray:
    """D^l(R) of the real harmonics, by least squares: Y_l(R u) = D Y_l(u) on
    random points (built from the harmonics alone, not from the CG)."""
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((n_pts, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    sl = slice(l * l, (l + 1) ** 2)
    A = sh(u, l)[:, sl]                       # [n, 2l+1]
    B = sh(u @ R.T, l)[:, sl]                 # rows Y(R u)
    Dt, *_ = np.linalg.lstsq(A, B, rcond=None)
    return Dt.T


def block_wigner(R: np.ndarray, irreps: str) -> np.ndarray:
    """Block-diagonal action on a feature row [D] (parity ignored: R proper)."""
    ir = parse_irreps(irreps)
    offs, D = block_offsets(ir)
    M = np.zeros((D, D))
    for (l, _), o in zip(ir, offs):
        M[o:o + 2 * l + 1, o:o + 2 * l + 1] = wigner_real(R, l)
    return M


def parity_signs(irreps: str) -> np.ndarray:
    ir = parse_irreps(irreps)
    return np.concatenate([np.full(2 * l + 1, float(p)) for l, p in ir])


def random_rotation(seed: int) -> np.ndarray:
    from scipy.spatial.transform import Rotation
    return Rotation.random(random_state=seed).as_matrix()


def within_tol(got, ref, rel=1e-5, abs_=1e-6):
    """max |got - ref| <= rel * max |ref| + abs_ (per output tensor)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return True, 0.0, 0.0
    err = float(np.max(np.abs(got - ref)))
    bound = rel * float(np.max(np.abs(ref))) + abs_
    return err <= bound, err, bound


def small_problem(N=12, E=40, C=8, L_in=2, L_sh=2, L_out=2, seed=0, irreps_in=None, irreps_out=None,
                  per_path=False):
    from oracle.conv import Problem
    from equivariant_gnn_message_edge_b200.workloads import natural_irreps
    rng = np.random.default_rng(seed)
    prob = Problem(irreps_in or natural_irreps(L_in), L_sh, irreps_out or natural_irreps(L_out), C,
                   per_path=per_path)
    senders = rng.integers(0, N, E).astype(np.int32)
    receivers = rng.integers(0, N, E).astype(np.int32)
    r = rng.standard_normal((E, 3)).astype(np.float32) * 2
    x = rng.standard_normal((N, prob.D_in, C)).astype(np.float32)
    w = rng.standard_normal((E, prob.P, C)).astype(np.float32)
    gy = rng.standard_normal((N, prob.D_out, C)).astype(np.float32)
    return prob, senders, receivers, r, x, w, gy
