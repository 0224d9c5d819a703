"""Pins for the oracle's convolution, forward and backward (no GPU).

e3j (arXiv 2609.35099), abstract / Table 1: the message-passing convolution,
forward and backward.  FlashCart (arXiv 2610.06409) App. B: the product must be
equivariant; §2: forces are energy gradients.  No page prints a worked
example, so every check here is a property the mathematics fixes:
equivariance (Wigner matrices built from the harmonics alone), parity,
invariance to edge order and node labels, an SpMM special case through SciPy,
bilinearity identities between forward and backward, finite differences for
dr, and agreement between two independent oracle implementations (NumPy
per-edge messages vs the C loops).
"""
import numpy as np
import pytest
import scipy.sparse as sp

from oracle import conv
from oracle.csr import csr
from oracle.sh import sh
from tests.helpers import block_wigner, parity_signs, random_rotation, small_problem

CASES = [dict(L_in=1, L_sh=2, L_out=2), dict(L_in=2, L_sh=2, L_out=2), dict(L_in=3, L_sh=3, L_out=3),
         dict(L_in=2, L_sh=1, L_out=3)]


@pytest.mark.parametrize("case", CASES)
def test_c_loops_match_bruteforce(case):
    N = 10
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=50, C=6, **case)
    y_ref = conv.forward_bruteforce(prob, N, s, rcv, r, x, w)
    dx_ref, dw_ref, dr_ref = conv.backward_bruteforce(prob, N, s, rcv, r, x, w, gy)
    y, dx, dw, dr = conv.full(prob, N, s, rcv, r, x, w, gy)
    for a, b in ((y, y_ref), (dx, dx_ref), (dw, dw_ref), (dr, dr_ref)):
        assert np.max(np.abs(a - b)) < 1e-11 * max(1.0, np.max(np.abs(b)))


def test_path_counts():
    from equivariant_gnn_message_edge_b200.workloads import natural_irreps
    assert conv.Problem("0e+1o", 2, natural_irreps(2), 4).P == 7
    assert conv.Problem(natural_irreps(2), 2, natural_irreps(2), 4).P == 11
    assert conv.Problem(natural_irreps(3), 3, natural_irreps(3), 4).P == 23


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_equivariance(case, seed):
    N = 9
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=40, C=5, seed=seed, **case)
    R = random_rotation(100 + seed)
    Din, Dout = block_wigner(R, prob.irreps_in), block_wigner(R, prob.irreps_out)
    y = conv.full(prob, N, s, rcv, r, x, w)
    xr = np.einsum("ab,nbc->nac", Din, x.astype(np.float64))
    rr = r.astype(np.float64) @ R.T
    # fp64 path through the NumPy oracle (C loops take fp32 inputs)
    y_rot = conv.forward_bruteforce(prob, N, s, rcv, rr, xr, w)
    assert np.max(np.abs(y_rot - np.einsum("ab,nbc->nac", Dout, y))) < 1e-10 * np.max(np.abs(y))


@pytest.mark.parametrize("case", CASES)
def test_parity(case):
    N = 8
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=30, C=4, **case)
    pin, pout = parity_signs(prob.irreps_in), parity_signs(prob.irreps_out)
    y = conv.forward_bruteforce(prob, N, s, rcv, r, x, w)
    y_inv = conv.forward_bruteforce(prob, N, s, rcv, -r.astype(np.float64), pin[None, :, None] * x, w)
    assert np.max(np.abs(y_inv - pout[None, :, None] * y)) < 1e-12 * np.max(np.abs(y))


def test_edge_order_and_relabel_invariance():
    N = 11
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=60, C=4)
    y, dx, dw, dr = conv.full(prob, N, s, rcv, r, x, w, gy)
    rng = np.random.default_rng(3)
    q = rng.permutation(len(s))                     # shuffle edges
    y2, dx2, dw2, dr2 = conv.full(prob, N, s[q], rcv[q], r[q], x, w[q], gy)
    assert np.max(np.abs(y2 - y)) < 1e-12 * np.max(np.abs(y))
    assert np.max(np.abs(dx2 - dx)) < 1e-12 * np.max(np.abs(dx))
    assert np.max(np.abs(dw2 - dw[q])) < 1e-12 * np.max(np.abs(dw))
    assert np.max(np.abs(dr2 - dr[q])) < 1e-12 * np.max(np.abs(dr))
    pi = rng.permutation(N).astype(np.int32)        # relabel nodes: new id = pi[old]
    inv = np.argsort(pi)
    y3 = conv.full(prob, N, pi[s], pi[rcv], r, x[inv], w)
    assert np.max(np.abs(y3[pi] - y)) < 1e-12 * np.max(np.abs(y))


def test_lsh0_is_weighted_spmm():
    """L_sh = 0: every path is l x 0 -> l with C = delta and Y_0 = 1, so
    y[:, l-block, :, c] = A_{p,c} x with A_{p,c}[i, j] = sum of w[e,p,c] over
    edges j -> i: a sparse matrix product (SciPy)."""
    N, E, C = 13, 70, 3
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=E, C=C, L_in=2, L_sh=0, L_out=2)
    y = conv.full(prob, N, s, rcv, r, x, w)
    ref = np.zeros_like(y)
    for p, q in enumerate(prob.paths):
        d = 2 * q["l1"] + 1
        for c in range(C):
            A = sp.csr_matrix((w[:, p, c].astype(np.float64), (rcv, s)), shape=(N, N))
            ref[:, q["off3"]:q["off3"] + d, c] += A @ x[:, q["off1"]:q["off1"] + d, c].astype(np.float64)
    assert np.max(np.abs(y - ref)) < 1e-12 * np.max(np.abs(ref))


@pytest.mark.parametrize("case", CASES)
def test_bilinearity(case):
    """y is linear in x and in w, so <gy, y> = <w, dw> = <x, dx>."""
    N = 10
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=45, C=5, **case)
    y, dx, dw, dr = conv.full(prob, N, s, rcv, r, x, w, gy)
    a = float((gy * y).sum())
    b = float((w * dw).sum())
    c = float((x * dx).sum())
    assert abs(a - b) < 1e-10 * abs(a) and abs(a - c) < 1e-10 * abs(a)


@pytest.mark.parametrize("case", CASES)
def test_dr_finite_differences(case):
    N = 7
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=20, C=3, **case)
    r = r.astype(np.float64)
    dr = conv.backward_bruteforce(prob, N, s, rcv, r, x, w, gy)[2]
    h = 1e-6
    for e in range(0, len(s), 3):
        for j in range(3):
            rp, rm = r.copy(), r.copy()
            rp[e, j] += h
            rm[e, j] -= h
            fp = float((gy * conv.forward_bruteforce(prob, N, s, rcv, rp, x, w)).sum())
            fm = float((gy * conv.forward_bruteforce(prob, N, s, rcv, rm, x, w)).sum())
            fd = (fp - fm) / (2 * h)
            assert abs(fd - dr[e, j]) < 1e-6 * max(1.0, abs(dr[e, j]))


def test_dr_radial_orthogonality_and_rotation():
    N = 9
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=40, C=4)
    r = r.astype(np.float64)
    _, _, dr = conv.backward_bruteforce(prob, N, s, rcv, r, x, w, gy)
    assert np.max(np.abs((dr * r).sum(1))) < 1e-11 * np.max(np.abs(dr))
    R = random_rotation(5)
    Din, Dout = block_wigner(R, prob.irreps_in), block_wigner(R, prob.irreps_out)
    xr = np.einsum("ab,nbc->nac", Din, x.astype(np.float64))
    gyr = np.einsum("ab,nbc->nac", Dout, gy.astype(np.float64))
    _, _, dr_rot = conv.backward_bruteforce(prob, N, s, rcv, r @ R.T, xr, w, gyr)
    assert np.max(np.abs(dr_rot - dr @ R.T)) < 1e-10 * np.max(np.abs(dr))


def test_zero_length_isolated_and_empty():
    N = 6
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=12, C=4)
    r[0] = 0.0
    rcv = np.where(rcv == 5, 4, rcv).astype(np.int32)      # node 5 receives nothing
    s = np.where(s == 3, 2, s).astype(np.int32)            # node 3 sends nothing
    y, dx, dw, dr = conv.full(prob, N, s, rcv, r, x, w, gy)
    assert np.all(dr[0] == 0.0)
    assert np.all(y[5] == 0.0) and np.all(dx[3] == 0.0)
    # edge 0 still contributes through Y_0 = 1: only l2 = 0 paths act
    Y = sh(r[:1], prob.L_sh)
    assert Y[0, 0] == 1.0 and np.all(Y[0, 1:] == 0.0)
    # no edges at all
    e0 = np.zeros(0, np.int32)
    y0, dx0, dw0, dr0 = conv.full(prob, N, e0, e0, np.zeros((0, 3), np.float32), x,
                                  np.zeros((0, prob.P, prob.C), np.float32), gy)
    assert np.all(y0 == 0) and np.all(dx0 == 0) and dw0.shape == (0, prob.P, prob.C) and dr0.shape == (0, 3)


def test_row_sampling_matches_full():
    N = 15
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=70, C=4)
    rp, rperm = csr(rcv, N)
    sp_, sperm = csr(s, N)
    Y = sh(r, prob.L_sh)
    y = conv.forward(prob, rp, rperm, s, Y, x, w)
    rows = np.array([3, 0, 14, 7], np.int32)
    assert np.array_equal(conv.forward(prob, rp, rperm, s, Y, x, w, rows=rows), y[rows])
    dx = conv.backward_dx(prob, sp_, sperm, rcv, Y, gy, w)
    assert np.array_equal(conv.backward_dx(prob, sp_, sperm, rcv, Y, gy, w, rows=rows), dx[rows])


def test_csr_definition():
    rng = np.random.default_rng(4)
    N, E = 20, 300
    keys = rng.integers(0, N, E).astype(np.int32)
    ptr, perm = csr(keys, N)
    # brute force: walk the keys in order and bucket them
    buckets = [[] for _ in range(N)]
    for e, k in enumerate(keys):
        buckets[k].append(e)
    assert list(perm) == [e for b in buckets for e in b]
    assert list(ptr) == list(np.cumsum([0] + [len(b) for b in buckets]))
    with pytest.raises(ValueError):
        csr(np.array([0, N], np.int32), N)
