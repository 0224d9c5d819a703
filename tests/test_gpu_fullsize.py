"""Full-size workloads on the GPU, in the launch configuration bench.py times,
checked against the oracle on sampled outputs (needs a B200).

lmax=2: N=32768, C=128, in-degree Poisson(45), E ~ 1.47M, P=11 (8.3 GB of w);
lmax=3: N=16384, C=128, E ~ 737k, P=23.  The oracle (fp64 C loops) computes y
for 256 sampled receivers, dx for 256 sampled senders, dw and dr for those
receivers' in-edges; every tensor is also checked for non-finite values.
"""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import workloads as wl
from equivariant_gnn_message_edge_b200.conv import EqConv
from oracle import conv as oconv
from oracle.csr import csr
from oracle.sh import sh, sh_grad
from tests.gpu_common import assert_close, to_dev

pytestmark = pytest.mark.gpu

N_SAMPLE = 256


def run_case(name):
    W = wl.WORKLOADS[name]
    s, rcv, r = wl.make_graph(W)
    E = len(s)
    prob = oconv.Problem(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    x = wl.features(W.N, prob.D_in, W.C, wl.SEED_X)
    gy = wl.features(W.N, prob.D_out, W.C, wl.SEED_GY)
    w = wl.weights(E, prob.P, W.C)

    conv = EqConv(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    g = conv.graph(to_dev(s), to_dev(rcv), W.N)
    xd, rd, gd = to_dev(x), to_dev(r), to_dev(gy)
    wd = to_dev(w)
    y = conv.forward_raw(g, xd, rd, wd)
    torch.cuda.synchronize()

    rng = np.random.default_rng(77)
    rows = np.sort(rng.choice(W.N, N_SAMPLE, replace=False)).astype(np.int32)
    senders_rows = np.sort(rng.choice(W.N, N_SAMPLE, replace=False)).astype(np.int32)
    rp, rperm = csr(rcv, W.N)
    sp, sperm = csr(s, W.N)
    assert np.array_equal(g.recv_ptr.cpu().numpy(), rp)
    assert np.array_equal(g.send_ptr.cpu().numpy(), sp)
    assert np.array_equal(g.send_perm[:E].cpu().numpy(), sperm)
    assert np.array_equal(g.recv_perm[:E].cpu().numpy(), rperm)
    Y = sh(r, W.L_sh)
    y_ref = oconv.forward(prob, rp, rperm, s, Y, x, w, rows=rows)
    y_rows = y[torch.from_numpy(rows).long().cuda()].cpu().numpy()
    assert_close("y(sampled)", y_rows, y_ref)
    assert torch.isfinite(y).all()

    edges = np.concatenate([rperm[rp[i]:rp[i + 1]] for i in rows]).astype(np.int32)
    dx_ref = oconv.backward_dx(prob, sp, sperm, rcv, Y, gy, w, rows=senders_rows)
    dw_ref, gY_ref = oconv.backward_edges(prob, s, rcv, Y, x, gy, w, edges=edges)
    J = sh_grad(r[edges], W.L_sh)
    dr_ref = np.einsum("ekj,ek->ej", J, gY_ref)
    del y, wd
    for det in (True, False):
        wd = to_dev(w)
        dx, dw, dr = conv.backward_raw(g, xd, rd, wd, gd, deterministic=det)
        torch.cuda.synchronize()
        tag = "det" if det else "atomic"
        assert_close(f"dx(sampled,{tag})", dx[torch.from_numpy(senders_rows).long().cuda()].cpu().numpy(), dx_ref)
        ed = torch.from_numpy(edges).long().cuda()
        assert_close(f"dw(sampled,{tag})", dw[ed].cpu().numpy(), dw_ref)
        assert_close(f"dr(sampled,{tag})", dr[ed].cpu().numpy(), dr_ref)
        assert torch.isfinite(dx).all() and torch.isfinite(dw).all() and torch.isfinite(dr).all()
        del dx, dw, dr, wd
        torch.cuda.empty_cache()


def test_fullsize_lmax2_sampled():
    run_case("lmax2")


def test_fullsize_lmax3_sampled():
    run_case("lmax3")


def run_double_backward_case(name, n_sample=64):
    """Double backward at full size: g_gy on sampled receivers, g_x on
    sampled senders, g_w and g_r on all their edges, against the oracle run
    on exactly those edges (which hold every term of the sampled rows)."""
    from oracle.dbl import double_backward_bruteforce
    W = wl.WORKLOADS[name]
    s, rcv, r = wl.make_graph(W)
    E = len(s)
    prob = oconv.Problem(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    x = wl.features(W.N, prob.D_in, W.C, wl.SEED_X)
    gy = wl.features(W.N, prob.D_out, W.C, wl.SEED_GY)
    w = wl.weights(E, prob.P, W.C)
    rng = np.random.default_rng(2024)
    a = rng.standard_normal((W.N, prob.D_in, W.C), dtype=np.float32)
    q = rng.standard_normal((E, 3), dtype=np.float32)
    b = rng.standard_normal((E, prob.P, W.C), dtype=np.float32)

    conv = EqConv(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    g = conv.graph(to_dev(s), to_dev(rcv), W.N)
    out = conv.double_backward_raw(g, to_dev(x), to_dev(r), to_dev(w), to_dev(gy), to_dev(a), to_dev(b), to_dev(q))
    torch.cuda.synchronize()
    g_x, g_w, g_gy, g_r = out
    assert all(torch.isfinite(t).all() for t in out)

    rows = np.sort(rng.choice(W.N, n_sample, replace=False))
    srows = np.sort(rng.choice(W.N, n_sample, replace=False))
    rp, rperm = csr(rcv, W.N)
    sp, sperm = csr(s, W.N)
    edges = np.unique(np.concatenate([rperm[rp[i]:rp[i + 1]] for i in rows] +
                                     [sperm[sp[j]:sp[j + 1]] for j in srows])).astype(np.int64)
    ref_x, ref_w, ref_gy, ref_r = double_backward_bruteforce(prob, W.N, s[edges], rcv[edges], r[edges], x, w[edges],
                                                             gy, a, b[edges], q[edges])
    ed = torch.from_numpy(edges).cuda()
    assert_close("g_gy(sampled)", g_gy[torch.from_numpy(rows).cuda()].cpu().numpy(), ref_gy[rows])
    assert_close("g_x(sampled)", g_x[torch.from_numpy(srows).cuda()].cpu().numpy(), ref_x[srows])
    assert_close("g_w(sampled)", g_w[ed].cpu().numpy(), ref_w)
    assert_close("g_r(sampled)", g_r[ed].cpu().numpy(), ref_r)


def test_fullsize_double_backward_lmax2_sampled():
    run_double_backward_case("lmax2")


def test_fullsize_double_backward_lmax3_sampled():
    run_double_backward_case("lmax3")
