"""Node-local channel-diagonal product on the GPU against the oracle
(FlashCart, arXiv 2610.06409, §5 and App. B/D).

Through the C ABI: y, du, dv and dw element by element against the fp64
oracle for several (L, C) cases with ragged channel tails, summed and
per-path layouts, with and without weights; bitwise reproducibility of the
backward (dw is summed over nodes in a fixed order); the autograd wrapper;
empty inputs and plans the op does not cover.
"""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import binding as B
from equivariant_gnn_message_edge_b200.conv import EqConv, NodeProduct
from equivariant_gnn_message_edge_b200.workloads import natural_irreps
from oracle import conv as oconv
from oracle.nodeprod import node_product, node_product_backward
from tests.gpu_common import assert_close, to_dev

pytestmark = pytest.mark.gpu

# (L_u, L_v, L_out, C, N)
CASES = [(1, 1, 2, 36, 300), (2, 2, 2, 132, 1000), (3, 3, 3, 100, 400), (2, 1, 3, 64, 700), (0, 3, 3, 8, 50),
         (3, 0, 3, 16, 90)]


def _inputs(prob, N, Lv, seed):
    rng = np.random.default_rng(seed)
    f = lambda *sh: rng.standard_normal(sh).astype(np.float32)
    return f(N, prob.D_in, prob.C), f(N, (Lv + 1) ** 2, prob.C), f(prob.P, prob.C), f(N, prob.D_out, prob.C)


@pytest.mark.parametrize("per_path", [False, True])
@pytest.mark.parametrize("weighted", [True, False])
@pytest.mark.parametrize("case", CASES)
def test_node_product_matches_oracle(case, weighted, per_path):
    Lu, Lv, Lout, C, N = case
    prob = oconv.Problem(natural_irreps(Lu), Lv, natural_irreps(Lout), C, per_path=per_path)
    u, v, w, gy = _inputs(prob, N, Lv, seed=CASES.index(case))
    w = w if weighted else None
    op = NodeProduct(natural_irreps(Lu), Lv, natural_irreps(Lout), C, per_path=per_path)
    assert op.D_out == prob.D_out and op.path_rows == [q["off3"] for q in prob.paths]
    ud, vd, gd = to_dev(u), to_dev(v), to_dev(gy)
    wd = None if w is None else to_dev(w)
    y = op.forward_raw(ud, vd, wd)
    du, dv, dw = op.backward_raw(ud, vd, wd, gd, need_dw=True)
    torch.cuda.synchronize()
    assert_close("y", y.cpu().numpy(), node_product(prob, u, v, w))
    rdu, rdv, rdw = node_product_backward(prob, u, v, w, gy)
    assert_close("du", du.cpu().numpy(), rdu)
    assert_close("dv", dv.cpu().numpy(), rdv)
    assert_close("dw", dw.cpu().numpy(), rdw)
    du2, dv2, dw2 = op.backward_raw(ud, vd, wd, gd, need_dw=True)
    assert torch.equal(du, du2) and torch.equal(dv, dv2) and torch.equal(dw, dw2)   # bitwise


def test_node_product_autograd_and_edge_cases():
    op = NodeProduct(natural_irreps(2), 2, natural_irreps(2), 64)
    prob = oconv.Problem(natural_irreps(2), 2, natural_irreps(2), 64)
    u, v, w, gy = _inputs(prob, 200, 2, seed=9)
    ut, vt, wt = (to_dev(t).requires_grad_() for t in (u, v, w))
    y = op(ut, vt, wt)
    (y * to_dev(gy)).sum().backward()
    rdu, rdv, rdw = node_product_backward(prob, u, v, w, gy)
    assert_close("du", ut.grad.cpu().numpy(), rdu)
    assert_close("dv", vt.grad.cpu().numpy(), rdv)
    assert_close("dw", wt.grad.cpu().numpy(), rdw)
    z = torch.zeros((0, 9, 64), device="cuda")
    e = op.forward_raw(z, z)
    assert e.shape == (0, 9, 64)
    du0, dv0, dw0 = op.backward_raw(z, z, to_dev(w), z)
    assert du0.shape == (0, 9, 64) and torch.equal(dw0, torch.zeros_like(dw0))
    with pytest.raises(B.EqconvError) as err:       # both parities are not offered for this op
        B.eqconv_node_product_plan_create("0e+1o", 1, "0e+1o+1e", 8, B.EQCONV_OUT_ALL_PARITY)
    assert err.value.status == B.EQCONV_ERR_UNSUPPORTED
    conv = EqConv("0e+1o", 1, "0e+1o", 8)            # a convolution plan is not a node-product plan
    with pytest.raises(B.EqconvError) as err:
        conv_y = torch.zeros((1, 4, 8), device="cuda")
        B.eqconv_node_product(conv.plan, 1, conv_y, conv_y, None, conv_y)
    assert err.value.status == B.EQCONV_ERR_INVALID_ARG
