"""The water-box step as stated, on the fused radial path (needs a B200):
two stacked convolution layers with radial-MLP weights, an energy-like
readout E = <gy, y2>, and the gradient of E with respect to the 1503
positions (the forces, through both routes of every edge vector: the
harmonics and the radial weights) and to both layers' MLP weights, against
the oracle's chain (e3j page, Table 2 / Table 3: MACE(a) water box, 2 layers,
C = 128, L = 3, 8 Bessel functions, 5 A cutoff; FlashCart §2: forces are the
energy's gradient in the positions).
"""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import workloads as wl
from equivariant_gnn_message_edge_b200.conv import RadialEqConv
from oracle import conv as oconv
from oracle import radial as orad
from tests.gpu_common import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _oracle_layer(prob, N, s, rcv, r, x, params, rc, gy):
    """One layer's forward and backward through both routes of r."""
    d = np.linalg.norm(r.astype(np.float64), axis=1)
    w = orad.radial_weights(d, rc, params, prob.P, prob.C).astype(np.float32)
    if gy is None:
        return oconv.full(prob, N, s, rcv, r, x, w)
    y, dx, dw, dr_ang = oconv.full(prob, N, s, rcv, r, x, w, gy)
    g_d, g_W = orad.radial_weights_vjp(d, rc, params, dw)
    safe = np.where(d > 0, d, 1.0)
    dr = dr_ang + (g_d / safe)[:, None] * r.astype(np.float64) * (d > 0)[:, None]
    return y, dx, dr, g_W


def test_waterbox_step_forces_and_weight_gradients():
    cfg = wl.WATER_BOX
    ins = wl.natural_irreps(cfg["L"])
    C, N, rc, nb = cfg["C"], cfg["n_atoms"], cfg["cutoff"], cfg["n_bessel"]
    pos, s, rcv, shift, dummy = wl.water_box_system()
    pos32, shift32 = pos.astype(np.float32), shift.astype(np.float32)
    r = (pos32[s] - pos32[rcv]) + shift32                      # the same fp32 arithmetic as on the GPU
    prob = oconv.Problem(ins, cfg["L"], ins, C)
    params = [wl.radial_mlp_params(prob.P, C, cfg["hidden"], nb, seed=wl.SEED_W + 10 * k) for k in range(2)]
    x1 = wl.features(N, prob.D_in, C, wl.SEED_X)
    readout = wl.features(N, prob.D_out, C, wl.SEED_GY)
    avg = float((~dummy).sum()) / N

    # GPU: the fused radial path under torch autograd
    conv = RadialEqConv(ins, cfg["L"], ins, C, n_basis=nb, r_cut=rc)
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    p = to_dev(pos32).requires_grad_(True)
    Ws = [[to_dev(t).requires_grad_(True) for t in ps] for ps in params]
    sl, rl = to_dev(s).long(), to_dev(rcv).long()
    rv = p[sl] - p[rl] + to_dev(shift32)
    y1 = conv(g, to_dev(x1), rv, *Ws[0])
    y2 = conv(g, y1 / avg, rv, *Ws[1])
    e = (y2 * to_dev(readout)).sum()
    grads = torch.autograd.grad(e, [p] + Ws[0] + Ws[1])
    torch.cuda.synchronize()
    assert np.array_equal(rv.detach().cpu().numpy(), r)

    # oracle: the same chain in fp64 (layer inputs it derives rounded to fp32,
    # as the C loops take fp32 inputs)
    y1r = _oracle_layer(prob, N, s, rcv, r, x1, params[0], rc, None)
    x2r = (y1r / avg).astype(np.float32)
    y2r, dx2r, dr2r, gW2r = _oracle_layer(prob, N, s, rcv, r, x2r, params[1], rc, readout)
    gy1r = (dx2r / avg).astype(np.float32)
    _, _, dr1r, gW1r = _oracle_layer(prob, N, s, rcv, r, x1, params[0], rc, gy1r)
    dr = dr1r + dr2r
    dpos = np.zeros((N, 3))
    np.add.at(dpos, s, dr)
    np.add.at(dpos, rcv, -dr)

    assert_close("y1", y1.detach().cpu().numpy(), y1r)
    assert_close("y2", y2.detach().cpu().numpy(), y2r)
    assert_close("dE/dpos (forces)", grads[0].cpu().numpy(), dpos)
    for k, gWr in enumerate((gW1r, gW2r)):
        for i in range(3):
            assert_close(f"layer {k + 1} g_W{i + 1}", grads[1 + 3 * k + i].cpu().numpy(), gWr[i])
