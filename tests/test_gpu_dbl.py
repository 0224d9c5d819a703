"""Double backward (VJP of the backward) on the GPU against the oracle
(FlashCart, arXiv 2610.06409, §2 and §3 / App. C: VJP-of-VJP of weighted
bilinear products, needed to train on forces).

Through the C ABI: the four gradients of S = <a, dx> + <b, dw> + <q, dr>
element by element against the fp64 oracle, for several (L, C) cases with
ragged channel tails and zero-length edges; bitwise reproducibility; and
torch double differentiation (create_graph=True) through the autograd
wrapper.
"""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import binding as B
from equivariant_gnn_message_edge_b200.conv import EqConv
from equivariant_gnn_message_edge_b200.workloads import natural_irreps
from oracle import conv as oconv
from oracle.dbl import double_backward_bruteforce
from tests.gpu_common import assert_close, to_dev

pytestmark = pytest.mark.gpu

# (L_in, L_sh, L_out, C, N, E)
CASES = [
    (1, 2, 2, 36, 40, 700),
    (2, 2, 2, 132, 90, 2500),
    (2, 1, 3, 64, 50, 900),
    (3, 3, 3, 100, 64, 1500),
    (0, 3, 2, 8, 30, 400),
    (1, 0, 1, 16, 20, 200),
]


def _inputs(prob, N, E, seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(0, N, E).astype(np.int32)
    rcv = rng.integers(0, N, E).astype(np.int32)
    r = (rng.standard_normal((E, 3)) * 2).astype(np.float32)
    r[1] = 0.0
    f = lambda *shape: rng.standard_normal(shape).astype(np.float32)
    x, gy, a = f(N, prob.D_in, prob.C), f(N, prob.D_out, prob.C), f(N, prob.D_in, prob.C)
    w = (f(E, prob.P, prob.C) / np.sqrt(prob.P)).astype(np.float32)
    b, q = f(E, prob.P, prob.C), f(E, 3)
    return s, rcv, r, x, w, gy, a, b, q


def _run(conv, s, rcv, N, *arrays):
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    out = conv.double_backward_raw(g, *[to_dev(t) for t in arrays])
    torch.cuda.synchronize()
    assert B.eqconv_get_device_error(conv.plan) == B.EQCONV_OK
    return [t.cpu().numpy() for t in out]


@pytest.mark.parametrize("case", CASES)
def test_double_backward_matches_oracle(case):
    L_in, L_sh, L_out, C, N, E = case
    ins, outs = natural_irreps(L_in), natural_irreps(L_out)
    prob = oconv.Problem(ins, L_sh, outs, C)
    s, rcv, r, x, w, gy, a, b, q = _inputs(prob, N, E, seed=CASES.index(case))
    ref = double_backward_bruteforce(prob, N, s, rcv, r, x, w, gy, a, b, q)
    conv = EqConv(ins, L_sh, outs, C)
    got = _run(conv, s, rcv, N, x, r, w, gy, a, b, q)
    for name, gv, rv in zip(("g_x", "g_w", "g_gy", "g_r"), got, ref):
        assert_close(name, gv, rv)
    again = _run(conv, s, rcv, N, x, r, w, gy, a, b, q)
    for gv, av in zip(got, again):
        assert np.array_equal(gv, av)          # deterministic: bitwise


def test_double_backward_empty_and_unsupported():
    conv = EqConv("0e+1o", 2, "0e+1o+2e", 8)
    N = 5
    s = rcv = np.zeros(0, np.int32)
    prob = oconv.Problem("0e+1o", 2, "0e+1o+2e", 8)
    x = np.ones((N, prob.D_in, 8), np.float32)
    gy = np.ones((N, prob.D_out, 8), np.float32)
    w, b = np.zeros((0, prob.P, 8), np.float32), np.zeros((0, prob.P, 8), np.float32)
    r = q = np.zeros((0, 3), np.float32)
    g_x, g_w, g_gy, g_r = _run(conv, s, rcv, N, x, r, w, gy, x, b, q)
    assert np.all(g_x == 0) and np.all(g_gy == 0) and g_w.size == 0 and g_r.size == 0
    pp = EqConv("0e+1o", 2, "0e+1o+2e", 8, per_path=True)
    g = pp.graph(to_dev(np.zeros(1, np.int32)), to_dev(np.zeros(1, np.int32)), 1)
    t = lambda *sh: torch.zeros(sh, device="cuda")
    with pytest.raises(B.EqconvError) as e:
        pp.double_backward_raw(g, t(1, 4, 8), t(1, 3), t(1, pp.P, 8), t(1, pp.D_out, 8), t(1, 4, 8),
                               t(1, pp.P, 8), t(1, 3))
    assert e.value.status == B.EQCONV_ERR_UNSUPPORTED


def test_autograd_double_differentiation_matches_oracle():
    """Force-style training: dS/d(x, r, w) of S = <a, dx> + <q, dr> + <b, dw>
    where (dx, dr, dw) come from torch.autograd.grad(create_graph=True)."""
    L_in, L_sh, L_out, C, N, E = 2, 2, 2, 64, 40, 800
    ins = natural_irreps(2)
    prob = oconv.Problem(ins, L_sh, ins, C)
    s, rcv, r, x, w, gy, a, b, q = _inputs(prob, N, E, seed=77)
    conv = EqConv(ins, L_sh, ins, C)
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    xt, rt, wt = (to_dev(t).requires_grad_() for t in (x, r, w))
    y = conv(g, xt, rt, wt)
    dx, dr, dw = torch.autograd.grad((y * to_dev(gy)).sum(), (xt, rt, wt), create_graph=True)
    S = (dx * to_dev(a)).sum() + (dr * to_dev(q)).sum() + (dw * to_dev(b)).sum()
    g_x, g_r, g_w = torch.autograd.grad(S, (xt, rt, wt))
    ref_x, ref_w, _, ref_r = double_backward_bruteforce(prob, N, s, rcv, r, x, w, gy, a, b, q)
    assert_close("g_x", g_x.cpu().numpy(), ref_x)
    assert_close("g_w", g_w.cpu().numpy(), ref_w)
    assert_close("g_r", g_r.cpu().numpy(), ref_r)
