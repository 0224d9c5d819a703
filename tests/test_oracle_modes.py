"""Pins for the oracle's two output variants: both-parity outputs and
per-path-retained outputs (no GPU).

FlashCart (arXiv 2610.06409) App. B: a path is admissible when the triangle
rule holds and the parities multiply; opposite-parity products (an odd
l1 + l2 + l3) are the antisymmetric couplings such as the cross product.
App. D: the channel-diagonal product may keep each path's output or sum the
paths that land on the same irrep.

What pins them, independently of the oracle's own formulas:
* the (1, 1, 1) coupling is the cross product (closed form);
* equivariance under rotations (Wigner matrices from the harmonics alone) and
  the inversion signs of every output block, both-parity pseudo-tensors
  included;
* per-path outputs summed by output irrep give the summed layout, which the
  other oracle tests pin; its backward with gy copied into every path block
  gives the summed backward;
* the two oracle implementations (NumPy messages, C loops) agree.
"""
import numpy as np
import pytest

from equivariant_gnn_message_edge_b200.workloads import both_parity_irreps, natural_irreps
from oracle import conv
from oracle.cg import real_cg
from oracle.irreps import block_offsets, parse_irreps
from oracle.sh import sh
from tests.helpers import block_wigner, parity_signs, random_rotation, small_problem

BOTH_CASES = [dict(L_in=1, L_sh=1, L_out=1), dict(L_in=2, L_sh=2, L_out=2), dict(L_in=1, L_sh=3, L_out=3),
              dict(L_in=3, L_sh=2, L_out=3)]


def _both(case, **kw):
    return small_problem(irreps_out=both_parity_irreps(case["L_out"]), **case, **kw)


def test_both_parity_irreps_and_path_counts():
    assert both_parity_irreps(0) == "0e"
    assert both_parity_irreps(2) == "0e+1o+1e+2e+2o"
    assert both_parity_irreps(3) == "0e+1o+1e+2e+2o+3o+3e"
    p2 = conv.Problem(natural_irreps(2), 2, both_parity_irreps(2), 4)
    assert p2.P == 15 and p2.D_out == 17
    odd = [(q["l1"], q["l2"], q["l3"]) for q in p2.paths if (q["l1"] + q["l2"] + q["l3"]) % 2]
    assert odd == [(1, 1, 1), (1, 2, 2), (2, 1, 2), (2, 2, 1)]
    # natural-parity inputs never reach 0o: l3 = 0 needs l1 = l2
    p3 = conv.Problem(natural_irreps(3), 3, "0o+1e", 4)
    assert all(q["l3"] == 1 for q in p3.paths)


def test_odd_coupling_is_the_cross_product():
    """Real l = 1 components are ordered (y, z, x); the (1,1,1) coupling of
    two vectors is (u x v)/sqrt2 in that order, up to the canonical sign."""
    rng = np.random.default_rng(3)
    C = real_cg(1, 1, 1)
    perm = [1, 2, 0]                        # (x, y, z) -> (y, z, x)
    for _ in range(5):
        u, v = rng.standard_normal(3), rng.standard_normal(3)
        got = np.einsum("abk,a,b->k", C, u[perm], v[perm])
        want = np.cross(u, v)[perm] / np.sqrt(2.0)
        assert np.allclose(np.abs(got), np.abs(want), atol=1e-13)
        sign = np.sign(got @ want)
        assert np.max(np.abs(got - sign * want)) < 1e-13


@pytest.mark.parametrize("case", BOTH_CASES)
@pytest.mark.parametrize("per_path", [False, True])
def test_both_parity_equivariance_and_inversion(case, per_path):
    N = 9
    prob, s, rcv, r, x, w, gy = _both(case, N=N, E=40, C=5, seed=4, per_path=per_path)
    R = random_rotation(7)
    Din, Dout = block_wigner(R, prob.irreps_in), block_wigner(R, prob.layout_out)
    y = conv.forward_bruteforce(prob, N, s, rcv, r, x, w)
    xr = np.einsum("ab,nbc->nac", Din, x.astype(np.float64))
    y_rot = conv.forward_bruteforce(prob, N, s, rcv, r.astype(np.float64) @ R.T, xr, w)
    assert np.max(np.abs(y_rot - np.einsum("ab,nbc->nac", Dout, y))) < 1e-10 * np.max(np.abs(y))
    pin, pout = parity_signs(prob.irreps_in), parity_signs(prob.layout_out)
    y_inv = conv.forward_bruteforce(prob, N, s, rcv, -r.astype(np.float64), pin[None, :, None] * x, w)
    assert np.max(np.abs(y_inv - pout[None, :, None] * y)) < 1e-12 * np.max(np.abs(y))
    # the pseudo-tensor blocks (parity opposite to (-1)^l) are not all zero
    ir = parse_irreps(prob.layout_out)
    offs, _ = block_offsets(ir)
    pseudo = [(o, l) for (l, p), o in zip(ir, offs) if p != (-1) ** l]
    assert pseudo
    for o, l in pseudo:
        assert np.max(np.abs(y[:, o:o + 2 * l + 1])) > 1e-3 * np.max(np.abs(y))


def _fold(prob_pp, prob_sum, y_pp):
    """Sum per-path blocks into the summed layout."""
    outs = parse_irreps(prob_sum.irreps_out)
    offs, _ = block_offsets(outs)
    y = np.zeros(y_pp.shape[:-2] + (prob_sum.D_out, y_pp.shape[-1]))
    for q in prob_pp.paths:
        d3 = 2 * q["l3"] + 1
        y[..., offs[q["i3"]]:offs[q["i3"]] + d3, :] += y_pp[..., q["off3"]:q["off3"] + d3, :]
    return y


def _spread(prob_pp, prob_sum, gy):
    """Copy every output irrep's gy into each path block that lands on it."""
    offs, _ = block_offsets(parse_irreps(prob_sum.irreps_out))
    g = np.zeros(gy.shape[:-2] + (prob_pp.D_out, gy.shape[-1]))
    for q in prob_pp.paths:
        d3 = 2 * q["l3"] + 1
        g[..., q["off3"]:q["off3"] + d3, :] = gy[..., offs[q["i3"]]:offs[q["i3"]] + d3, :]
    return g


@pytest.mark.parametrize("outs", ["natural", "both"])
@pytest.mark.parametrize("case", BOTH_CASES)
def test_per_path_blocks_sum_to_the_summed_layout(case, outs):
    N = 10
    out = natural_irreps(case["L_out"]) if outs == "natural" else both_parity_irreps(case["L_out"])
    ps, s, rcv, r, x, w, gy = small_problem(N=N, E=50, C=6, seed=2, irreps_out=out, **case)
    pp = conv.Problem(ps.irreps_in, ps.L_sh, out, ps.C, per_path=True)
    assert pp.P == ps.P and pp.D_out == sum(2 * q["l3"] + 1 for q in pp.paths)
    y_s, dx_s, dw_s, dr_s = conv.full(ps, N, s, rcv, r, x, w, gy)
    gy_pp = _spread(pp, ps, gy.astype(np.float64)).astype(np.float32)
    y_p, dx_p, dw_p, dr_p = conv.full(pp, N, s, rcv, r, x, w, gy_pp)
    tol = 1e-11
    assert np.max(np.abs(_fold(pp, ps, y_p) - y_s)) < tol * np.max(np.abs(y_s))
    for a, b in ((dx_p, dx_s), (dw_p, dw_s), (dr_p, dr_s)):
        assert np.max(np.abs(a - b)) < tol * max(1.0, np.max(np.abs(b)))


@pytest.mark.parametrize("case", BOTH_CASES[:3])
@pytest.mark.parametrize("per_path", [False, True])
def test_c_loops_match_bruteforce_in_both_layouts(case, per_path):
    N = 10
    prob, s, rcv, r, x, w, gy = _both(case, N=N, E=50, C=6, seed=9, per_path=per_path)
    y_ref = conv.forward_bruteforce(prob, N, s, rcv, r, x, w)
    dx_ref, dw_ref, dr_ref = conv.backward_bruteforce(prob, N, s, rcv, r, x, w, gy)
    y, dx, dw, dr = conv.full(prob, N, s, rcv, r, x, w, gy)
    for a, b in ((y, y_ref), (dx, dx_ref), (dw, dw_ref), (dr, dr_ref)):
        assert np.max(np.abs(a - b)) < 1e-11 * max(1.0, np.max(np.abs(b)))


def test_odd_paths_give_nonzero_pseudotensors():
    """A 1o x Y_1 -> 1e message is x x r-hat scaled: it vanishes for x
    parallel to r and not otherwise."""
    prob = conv.Problem("1o", 1, "1e", 1)
    assert [(q["l1"], q["l2"], q["l3"]) for q in prob.paths] == [(1, 1, 1)]
    r = np.array([[0.3, -1.2, 0.7]], dtype=np.float32)
    Y1 = sh(r, 1)[0, 1:4]                       # sqrt3 * (y, z, x) of r-hat
    s = np.zeros(1, np.int32)
    w = np.ones((1, 1, 1), np.float32)
    par = (Y1 / np.sqrt(3.0)).astype(np.float32).reshape(1, 3, 1)
    y = conv.forward_bruteforce(prob, 1, s, s, r, par, w)
    assert np.max(np.abs(y)) < 1e-7
    perp = np.array([1.2, 0.3, 0.0], np.float32).reshape(1, 3, 1)     # (y, z, x) components
    y = conv.forward_bruteforce(prob, 1, s, s, r, perp, w)
    u = r[0] / np.linalg.norm(r[0])
    xv = np.array([0.0, 1.2, 0.3])                                     # (x, y, z)
    want = np.sqrt(3.0) * np.cross(xv, u)[[1, 2, 0]] / np.sqrt(2.0)
    assert np.allclose(np.abs(y[0, :, 0]), np.abs(want), atol=1e-6)
