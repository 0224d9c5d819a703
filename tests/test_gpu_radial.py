"""Radial weights on the tensor cores (eqconv_radial_weights) against the
oracle's radial MLP (needs a B200).

w[e, p, c] = u(|r_e|) * (silu(silu(b(|r_e|) W1) W2) W3)[p*C + c] with the
Bessel basis b and the C2 polynomial envelope u (FlashCart App. B / App. E;
e3j Table 3: 8 Bessel functions, 5 A cutoff).  The last layer runs as fp16
hi/lo products with fp32 accumulation in tensor memory; the result must match
the fp64 oracle within the convolution's tolerance, at sizes that span
several 128-row and 64-edge tiles with ragged tails, for edges at, beyond and
on zero length, and for weights of very different scales.
"""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import binding as B
from equivariant_gnn_message_edge_b200 import workloads as wl
from equivariant_gnn_message_edge_b200.conv import EqConv
from oracle import radial as orad
from tests.gpu_common import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _edges(E, rc, seed):
    rng = np.random.default_rng(seed)
    d = rng.standard_normal((E, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    length = rng.uniform(0.3, 1.1 * rc, size=E)      # some beyond the cutoff
    r = d * length[:, None]
    if E >= 4:
        r[0] = 0.0                                   # zero length
        r[1] = [rc, 0.0, 0.0]                        # exactly at the cutoff: u = 0
        r[2] = [0.0, 0.0, 1e-3]                      # very short
    return r.astype(np.float32)


def _gpu_weights(conv, r, params, n_basis, rc):
    E = r.shape[0]
    ws_n = B.eqconv_radial_workspace_bytes(conv.plan, E)
    ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
    w = torch.full((max(E, 1), conv.P, conv.C), float("nan"), device="cuda")
    W1, W2, W3 = (to_dev(p) for p in params)
    B.eqconv_radial_weights(conv.plan, E, to_dev(r), W1, W2, W3, n_basis, rc, w, ws, ws_n)
    torch.cuda.synchronize()
    assert B.eqconv_get_device_error(conv.plan) == B.EQCONV_OK
    return w[:E].cpu().numpy()


@pytest.mark.parametrize("L,C,E", [(1, 32, 1), (1, 32, 65), (2, 128, 1000), (2, 32, 333), (3, 64, 700),
                                   (3, 128, 129)])
def test_radial_weights_match_oracle(L, C, E):
    ins = wl.natural_irreps(L)
    conv = EqConv(ins, L, ins, C)
    rc, nb = 5.0, 8
    r = _edges(E, rc, seed=E + C)
    params = wl.radial_mlp_params(conv.P, C, 64, nb, seed=7 + L)
    got = _gpu_weights(conv, r, params, nb, rc)
    want = orad.radial_weights(np.linalg.norm(r.astype(np.float64), axis=1), rc, params, conv.P, C)
    assert_close(f"w L={L} C={C} E={E}", got, want)
    d = np.linalg.norm(r.astype(np.float64), axis=1)
    assert np.all(got[d >= rc * (1 + 1e-6)] == 0.0), "weights beyond the cutoff must be exactly zero"


@pytest.mark.parametrize("scale", [1e-4, 1e3])
def test_radial_weights_scale_robust(scale):
    """The power-of-two scaling keeps the fp16 halves in range for weights
    far from unit size."""
    conv = EqConv("0e+1o+2e", 2, "0e+1o+2e", 64)
    rc, nb = 5.0, 8
    r = _edges(500, rc, seed=3)
    params = wl.radial_mlp_params(conv.P, 64, 64, nb, seed=11)
    params = [params[0], params[1] * np.float32(scale), params[2] * np.float32(1.0 / scale)]
    got = _gpu_weights(conv, r, params, nb, rc)
    want = orad.radial_weights(np.linalg.norm(r.astype(np.float64), axis=1), rc, params, conv.P, 64)
    assert_close(f"w scale {scale}", got, want)


def test_radial_weights_water_box():
    """The water box's own edges and MLP (dummy edges at the cutoff get 0)."""
    cfg = wl.WATER_BOX
    ins = wl.natural_irreps(cfg["L"])
    conv = EqConv(ins, cfg["L"], ins, cfg["C"])
    s, rcv, r, dummy = wl.water_box_graph()
    params = wl.radial_mlp_params(conv.P, cfg["C"], cfg["hidden"], cfg["n_bessel"])
    got = _gpu_weights(conv, r, params, cfg["n_bessel"], cfg["cutoff"])
    ref = orad.radial_weights(np.linalg.norm(r.astype(np.float64), axis=1), cfg["cutoff"], params, conv.P, cfg["C"])
    assert_close("water box w", got, ref)
    assert np.all(got[dummy] == 0.0)


# ------------------------------------------------ fused forward (radial on chip)

def _poisson_case(N, mean_deg, seed):
    rng = np.random.default_rng(seed)
    deg = rng.poisson(mean_deg, size=N)
    deg[::7] = 0                                         # receivers with no in-edges
    rcv = np.repeat(np.arange(N, dtype=np.int32), deg)
    snd = rng.integers(0, N, size=rcv.size).astype(np.int32)
    r = _edges(rcv.size, 5.0, seed + 1)
    return snd, rcv, r


def _fused_forward(conv, N, s, rcv, r, x, params, nb, rc):
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    ws_n = B.eqconv_forward_radial_workspace_bytes(conv.plan, N, len(s))
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device="cuda")
    y = torch.full((N, conv.D_out, conv.C), float("nan"), device="cuda")
    W1, W2, W3 = (to_dev(p) for p in params)
    B.eqconv_forward_radial(conv.plan, g.c, to_dev(x), to_dev(r), W1, W2, W3, nb, rc, y, ws, ws_n)
    torch.cuda.synchronize()
    assert B.eqconv_get_device_error(conv.plan) == B.EQCONV_OK
    return y.cpu().numpy()


def test_forward_radial_tiny_box_against_bruteforce():
    """The tiny box (0e+1o -> 0e+1o+2e, L_sh = 2) against the oracle's
    composition of the radial MLP with the per-edge message brute force."""
    from oracle import conv as oconv
    W = wl.WORKLOADS["tiny"]
    s, rcv, r = wl.make_graph(W)
    conv = EqConv(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    prob = oconv.Problem(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    x = wl.features(W.N, prob.D_in, W.C, wl.SEED_X)
    params = wl.radial_mlp_params(prob.P, W.C, 64, 8, seed=21)
    got = _fused_forward(conv, W.N, s, rcv, r, x, params, 8, 3.5)
    want = orad.conv_with_radial(prob, W.N, s, rcv, r, x, 3.5, params)
    assert_close("y (fused radial, tiny box)", got, want)


@pytest.mark.parametrize("L,C,N,per_path", [(1, 32, 300, False), (2, 64, 700, False), (2, 128, 517, True),
                                            (3, 64, 400, False), (3, 32, 129, True)])
def test_forward_radial_matches_oracle(L, C, N, per_path):
    """Several channel slices, one or two path groups (L = 3: 23 paths),
    ragged receiver ranges, receivers without edges, edges beyond the cutoff
    and of zero length; summed and per-path output layouts."""
    from oracle import conv as oconv
    ins = wl.natural_irreps(L)
    conv = EqConv(ins, L, ins, C, per_path=per_path)
    prob = oconv.Problem(ins, L, ins, C, per_path=per_path)
    s, rcv, r = _poisson_case(N, 12.0, seed=N + C)
    x = wl.features(N, prob.D_in, C, wl.SEED_X)
    rc, nb = 5.0, 8
    params = wl.radial_mlp_params(prob.P, C, 64, nb, seed=31 + L)
    got = _fused_forward(conv, N, s, rcv, r, x, params, nb, rc)
    w = orad.radial_weights(np.linalg.norm(r.astype(np.float64), axis=1), rc, params, prob.P, C).astype(np.float32)
    want = oconv.full(prob, N, s, rcv, r, x, w)
    assert_close(f"y (fused radial L={L} C={C} N={N} per_path={per_path})", got, want)


def test_forward_radial_no_edges_and_unsupported():
    conv = EqConv("0e+1o+2e", 2, "0e+1o+2e", 32)
    x = np.ones((5, 9, 32), np.float32)
    params = wl.radial_mlp_params(conv.P, 32, 64, 8)
    got = _fused_forward(conv, 5, np.zeros(0, np.int32), np.zeros(0, np.int32), np.zeros((0, 3), np.float32), x,
                         params, 8, 5.0)
    assert np.all(got == 0.0)
    odd = EqConv("0e+1o", 1, "0e+1o", 32)          # (1, 1, 1) is compiled; (2, 1, 2) is not
    assert B.eqconv_forward_radial_workspace_bytes(odd.plan, 10, 10) > 0
    other = EqConv("0e+1o+2e", 1, "0e+1o+2e", 32)
    assert B.eqconv_forward_radial_workspace_bytes(other.plan, 10, 10) == 0


# ----------------------------------------------- fused backward (radial on chip)

def _fused_backward(conv, N, s, rcv, r, x, params, nb, rc, gy):
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    E = len(s)
    ws_n = B.eqconv_backward_radial_workspace_bytes(conv.plan, N, E)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device="cuda")
    nan = float("nan")
    dx = torch.full((N, conv.D_in, conv.C), nan, device="cuda")
    dr = torch.full((max(E, 1), 3), nan, device="cuda")
    gW = [torch.full(tuple(p.shape), nan, device="cuda") for p in params]
    W1, W2, W3 = (to_dev(p) for p in params)
    B.eqconv_backward_radial(conv.plan, g.c, to_dev(x), to_dev(r), W1, W2, W3, nb, rc, to_dev(gy), dx, dr,
                             gW[0], gW[1], gW[2], ws, ws_n)
    torch.cuda.synchronize()
    assert B.eqconv_get_device_error(conv.plan) == B.EQCONV_OK
    return dx.cpu().numpy(), dr[:E].cpu().numpy(), [t.cpu().numpy() for t in gW]


def _oracle_backward(prob, N, s, rcv, r, x, params, rc, gy):
    """dx, dr (both routes of r) and the MLP weight gradients: the oracle's
    C-loop backward with w from the radial MLP, then the MLP's VJP."""
    from oracle import conv as oconv
    d = np.linalg.norm(r.astype(np.float64), axis=1)
    w = orad.radial_weights(d, rc, params, prob.P, prob.C).astype(np.float32)
    _, dx, dw, dr_ang = oconv.full(prob, N, s, rcv, r, x, w, gy)
    g_d, g_W = orad.radial_weights_vjp(d, rc, params, dw)
    safe = np.where(d > 0, d, 1.0)
    dr = dr_ang + (g_d / safe)[:, None] * r.astype(np.float64) * (d > 0)[:, None]
    return dx, dr, g_W


def test_backward_radial_tiny_box_against_bruteforce():
    from oracle import conv as oconv
    W = wl.WORKLOADS["tiny"]
    s, rcv, r = wl.make_graph(W)
    conv = EqConv(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    prob = oconv.Problem(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    x = wl.features(W.N, prob.D_in, W.C, wl.SEED_X)
    gy = wl.features(W.N, prob.D_out, W.C, wl.SEED_GY)
    params = wl.radial_mlp_params(prob.P, W.C, 64, 8, seed=21)
    dx, dr, gW = _fused_backward(conv, W.N, s, rcv, r, x, params, 8, 3.5, gy)
    _, dxr, drr, gWr = orad.conv_with_radial(prob, W.N, s, rcv, r, x, 3.5, params, gy=gy)
    assert_close("dx (fused radial, tiny box)", dx, dxr)
    assert_close("dr (fused radial, tiny box)", dr, drr)
    for i in range(3):
        assert_close(f"g_W{i + 1} (fused radial, tiny box)", gW[i], gWr[i])


@pytest.mark.parametrize("L,C,N,per_path", [(1, 32, 300, False), (2, 64, 700, False), (2, 128, 517, True),
                                            (3, 64, 400, False), (3, 32, 129, True)])
def test_backward_radial_matches_oracle(L, C, N, per_path):
    from oracle import conv as oconv
    ins = wl.natural_irreps(L)
    conv = EqConv(ins, L, ins, C, per_path=per_path)
    prob = oconv.Problem(ins, L, ins, C, per_path=per_path)
    s, rcv, r = _poisson_case(N, 12.0, seed=N + C + 5)
    x = wl.features(N, prob.D_in, C, wl.SEED_X)
    gy = wl.features(N, prob.D_out, C, wl.SEED_GY)
    rc, nb = 5.0, 8
    params = wl.radial_mlp_params(prob.P, C, 64, nb, seed=41 + L)
    dx, dr, gW = _fused_backward(conv, N, s, rcv, r, x, params, nb, rc, gy)
    dxr, drr, gWr = _oracle_backward(prob, N, s, rcv, r, x, params, rc, gy)
    tag = f"L={L} C={C} N={N} per_path={per_path}"
    assert_close(f"dx ({tag})", dx, dxr)
    assert_close(f"dr ({tag})", dr, drr)
    for i in range(3):
        assert_close(f"g_W{i + 1} ({tag})", gW[i], gWr[i])


def test_backward_radial_is_bitwise_reproducible():
    ins = "0e+1o+2e"
    conv = EqConv(ins, 2, ins, 64)
    N = 600
    s, rcv, r = _poisson_case(N, 20.0, seed=9)
    x = wl.features(N, 9, 64, wl.SEED_X)
    gy = wl.features(N, 9, 64, wl.SEED_GY)
    params = wl.radial_mlp_params(conv.P, 64, 64, 8, seed=3)
    a = _fused_backward(conv, N, s, rcv, r, x, params, 8, 5.0, gy)
    b = _fused_backward(conv, N, s, rcv, r, x, params, 8, 5.0, gy)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    for i in range(3):
        assert np.array_equal(a[2][i], b[2][i])
