"""Pins for the oracle's node-local channel-diagonal product (no GPU).

FlashCart (arXiv 2610.06409) §5, App. B and App. D: pairwise channel-diagonal
products of node features along admissible paths, with path retention or
weighted summation.  What pins the oracle, independently of its formula:
* closed forms: the (1,1,0) path is the dot product / sqrt3, the (1,1,1)
  path (both parities) the cross product / sqrt2, the (l,0,l) path the
  scalar multiple;
* rotation equivariance (Wigner matrices from the harmonics) and inversion
  signs, summed and per-path layouts;
* with v set to the harmonics of a direction in every channel, the product
  equals the convolution's forward on a graph of self-edges (the C-loop
  oracle, an independent implementation);
* the backward: y is linear in each of u, v and w, so finite differences in
  any direction are exact, and <gy,y> = <du,u> = <dv,v> = <dw,w>.
"""
import numpy as np
import pytest

from equivariant_gnn_message_edge_b200.workloads import both_parity_irreps, natural_irreps
from oracle import conv
from oracle.nodeprod import node_product, node_product_backward
from oracle.sh import sh
from tests.helpers import block_wigner, parity_signs, random_rotation

CASES = [(1, 1, 2), (2, 2, 2), (3, 3, 3), (2, 1, 3), (0, 3, 3), (3, 2, 1)]


def _setup(Lu, Lv, Lout, C=5, N=7, seed=0, per_path=False, all_parity=False):
    outs = both_parity_irreps(Lout) if all_parity else natural_irreps(Lout)
    prob = conv.Problem(natural_irreps(Lu), Lv, outs, C, per_path=per_path)
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((N, prob.D_in, C))
    v = rng.standard_normal((N, (Lv + 1) ** 2, C))
    w = rng.standard_normal((prob.P, C))
    gy = rng.standard_normal((N, prob.D_out, C))
    return prob, u, v, w, gy


def test_closed_forms():
    rng = np.random.default_rng(1)
    perm = [1, 2, 0]                                  # (x, y, z) -> (y, z, x)
    uc, vc = rng.standard_normal((6, 3)), rng.standard_normal((6, 3))
    u = np.zeros((6, 4, 1))
    v = np.zeros((6, 4, 1))
    u[:, 1:4, 0], v[:, 1:4, 0] = uc[:, perm], vc[:, perm]
    dot = conv.Problem("0e+1o", 1, "0e", 1)
    assert [(q["l1"], q["l2"], q["l3"]) for q in dot.paths] == [(0, 0, 0), (1, 1, 0)]
    y = node_product(dot, u, v)[:, 0, 0]
    assert np.allclose(np.abs(y), np.abs((uc * vc).sum(1)) / np.sqrt(3.0), atol=1e-13)
    cross = conv.Problem("1o", 1, "1e", 1)
    y = node_product(cross, u[:, 1:4], v)[:, :, 0]
    want = np.cross(uc, vc)[:, perm] / np.sqrt(2.0)
    sgn = np.sign((y * want).sum())
    assert np.max(np.abs(y - sgn * want)) < 1e-13
    scal = conv.Problem("0e+1o+2e", 0, "0e+1o+2e", 3)
    uu, vv, ww = rng.standard_normal((4, 9, 3)), rng.standard_normal((4, 1, 3)), rng.standard_normal((3, 3))
    assert np.max(np.abs(node_product(scal, uu, vv, ww) - np.repeat(ww, [1, 3, 5], axis=0) * uu * vv)) < 1e-13


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("layout", ["summed", "per_path", "both"])
def test_equivariance_and_inversion(case, layout):
    prob, u, v, w, _ = _setup(*case, seed=2, per_path=layout == "per_path", all_parity=layout == "both")
    R = random_rotation(5)
    Du = block_wigner(R, prob.irreps_in)
    Dv = block_wigner(R, natural_irreps(case[1]))
    Dy = block_wigner(R, prob.layout_out)
    y = node_product(prob, u, v, w)
    y_rot = node_product(prob, np.einsum("ab,nbc->nac", Du, u), np.einsum("ab,nbc->nac", Dv, v), w)
    assert np.max(np.abs(y_rot - np.einsum("ab,nbc->nac", Dy, y))) < 1e-10 * np.max(np.abs(y))
    pu, pv, py = parity_signs(prob.irreps_in), parity_signs(natural_irreps(case[1])), parity_signs(prob.layout_out)
    y_inv = node_product(prob, pu[None, :, None] * u, pv[None, :, None] * v, w)
    assert np.max(np.abs(y_inv - py[None, :, None] * y)) < 1e-12 * np.max(np.abs(y))


@pytest.mark.parametrize("case", CASES)
def test_harmonic_v_equals_the_convolution_on_self_edges(case):
    Lu, Lv, Lout = case
    prob, u, _, w, _ = _setup(*case, seed=3)
    N, C = u.shape[0], prob.C
    r = np.random.default_rng(4).standard_normal((N, 3)).astype(np.float32)
    v = np.repeat(sh(r, Lv)[:, :, None], C, axis=2)
    idx = np.arange(N, dtype=np.int32)
    we = np.broadcast_to(w, (N, prob.P, C)).astype(np.float32)
    y_conv = conv.full(prob, N, idx, idx, r, u.astype(np.float32), we)
    y = node_product(prob, u.astype(np.float32), v, we[0])
    assert np.max(np.abs(y - y_conv)) < 1e-9 * np.max(np.abs(y_conv))


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("per_path", [False, True])
def test_backward_is_exact_directional_derivative(case, per_path):
    prob, u, v, w, gy = _setup(*case, seed=6, per_path=per_path)
    du, dv, dw = node_product_backward(prob, u, v, w, gy)
    S = lambda uu, vv, ww: float((gy * node_product(prob, uu, vv, ww)).sum())
    s0 = S(u, v, w)
    rng = np.random.default_rng(7)
    for name, g in (("u", du), ("v", dv), ("w", dw)):
        d = rng.standard_normal(g.shape)
        args = dict(u=u, v=v, w=w)
        args[name] = args[name] + d
        lhs = S(args["u"], args["v"], args["w"]) - s0     # linear in each argument: exact
        assert abs(lhs - (g * d).sum()) < 1e-10 * max(1.0, abs(lhs))
    for t, g in ((u, du), (v, dv), (w, dw)):
        assert abs((t * g).sum() - s0) < 1e-10 * max(1.0, abs(s0))
