"""The MACE(a)-shaped water box (e3j page, Table 2 and Table 3 setting), two
stacked convolution layers forward and backward, checked in full against the
oracle (needs a B200).

1503 atoms by random sequential addition (minimum distance 0.9 A) in a 25 A
periodic cube, cutoff 5 A (about 50 neighbours), 10% zero-weight dummy edges
(i -> i, r = (cutoff, 0, 0)); C = 128, L_in = L_sh = L_out = 3; radial weights
from a seeded Bessel(8) x polynomial envelope x 2-layer MLP.  Layer 2 takes
y1 / <degree>.  The oracle computes its own chain in fp64 from the same inputs.
"""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import workloads as wl
from equivariant_gnn_message_edge_b200.conv import EqConv
from oracle import conv as oconv
from tests.gpu_common import assert_close, to_dev

pytestmark = pytest.mark.gpu


def test_waterbox_two_layers_forward_backward():
    cfg = wl.WATER_BOX
    ins = wl.natural_irreps(cfg["L"])
    C, N = cfg["C"], cfg["n_atoms"]
    pos = wl.random_sequential_packing(N, cfg["box"], cfg["min_dist"])
    s, rcv, r, dummy = wl.padded_box_graph(pos, cfg["box"], cfg["cutoff"], cfg["pad"])
    prob = oconv.Problem(ins, cfg["L"], ins, C)
    w1 = wl.radial_weights(r, cfg["cutoff"], wl.radial_mlp_params(prob.P, C, seed=wl.SEED_W), prob.P, C, dummy)
    w2 = wl.radial_weights(r, cfg["cutoff"], wl.radial_mlp_params(prob.P, C, seed=wl.SEED_W + 10), prob.P, C, dummy)
    x1 = wl.features(N, prob.D_in, C, wl.SEED_X)
    gy2 = wl.features(N, prob.D_out, C, wl.SEED_GY)
    avg = float((~dummy).sum()) / N

    # oracle chain: fp64 accumulation; the layer inputs it derives (x2, gy1)
    # are rounded to fp32 like the GPU's, since the C loops take fp32 inputs
    y1r = oconv.full(prob, N, s, rcv, r, x1, w1)
    x2r = (y1r / avg).astype(np.float32)
    y2r, dx2r, dw2r, dr2r = oconv.full(prob, N, s, rcv, r, x2r, w2, gy2)
    gy1r = (dx2r / avg).astype(np.float32)
    _, dx1r, dw1r, dr1r = oconv.full(prob, N, s, rcv, r, x1, w1, gy1r)

    conv = EqConv(ins, cfg["L"], ins, C)
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    rd, w1d, w2d = to_dev(r), to_dev(w1), to_dev(w2)
    y1 = conv.forward_raw(g, to_dev(x1), rd, w1d)
    x2 = y1 / avg
    y2 = conv.forward_raw(g, x2, rd, w2d)
    for det in (True, False):
        dx2, dw2, dr2 = conv.backward_raw(g, x2, rd, w2d, to_dev(gy2), deterministic=det)
        dx1, dw1, dr1 = conv.backward_raw(g, to_dev(x1), rd, w1d, dx2 / avg, deterministic=det)
        torch.cuda.synchronize()
        tag = "det" if det else "atomic"
        assert_close("y1", y1.cpu().numpy(), y1r)
        assert_close("y2", y2.cpu().numpy(), y2r)
        assert_close(f"dx2 {tag}", dx2.cpu().numpy(), dx2r)
        assert_close(f"dw2 {tag}", dw2.cpu().numpy(), dw2r)
        assert_close(f"dr2 {tag}", dr2.cpu().numpy(), dr2r)
        assert_close(f"dx1 {tag}", dx1.cpu().numpy(), dx1r)
        assert_close(f"dw1 {tag}", dw1.cpu().numpy(), dw1r)
        assert_close(f"dr1 {tag}", dr1.cpu().numpy(), dr1r)
        # dummy edges (w = 0) contribute nothing, so their dr is zero
        assert np.all(np.abs(dr1.cpu().numpy()[dummy]) <= 1e-6 * np.abs(dr1r).max() + 1e-6)
