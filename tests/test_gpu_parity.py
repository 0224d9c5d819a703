"""CUDA path vs oracle, element by element, on seeded inputs (needs a B200).

Tolerance per output tensor (y, dx, dw, dr): max|gpu - ref| <= 1e-5 max|ref|
+ 1e-6 with ref the fp64 oracle; CSR offsets and permutations bit-exact;
deterministic mode bitwise identical run to run.
"""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import binding as B
from equivariant_gnn_message_edge_b200 import workloads as wl
from equivariant_gnn_message_edge_b200.conv import EqConv
from oracle.sh import sh
from tests.gpu_common import assert_close, check_all, check_csr, oracle_full, run_gpu, to_dev

pytestmark = pytest.mark.gpu

NAT = wl.natural_irreps


def random_case(N, E, C, L_in, L_sh, L_out, seed, sorted_recv=False):
    rng = np.random.default_rng(seed)
    P = len(B.eqconv_enumerate_paths(NAT(L_in), L_sh, NAT(L_out)))
    senders = rng.integers(0, N, E).astype(np.int32)
    receivers = rng.integers(0, N, E).astype(np.int32)
    if sorted_recv:
        receivers = np.sort(receivers).astype(np.int32)
    r = (rng.standard_normal((E, 3)) * 2).astype(np.float32)
    x = rng.standard_normal((N, (L_in + 1) ** 2, C)).astype(np.float32)
    w = (rng.standard_normal((E, P, C)) / np.sqrt(P)).astype(np.float32)
    gy = rng.standard_normal((N, (L_out + 1) ** 2, C)).astype(np.float32)
    return senders, receivers, r, x, w, gy


# ------------------------------------------------------------------ harmonics

@pytest.mark.parametrize("L", [0, 1, 2, 3])
def test_spherical_harmonics(L):
    rng = np.random.default_rng(L)
    r = (rng.standard_normal((5000, 3)) * rng.uniform(0.1, 10, (5000, 1))).astype(np.float32)
    r[0] = 0.0
    r[1] = [1e-20, 0, 0]
    r[2] = [0, 0, 3.0]
    r[3] = [0, 0, -2.0]
    conv = EqConv(NAT(min(L, 3)), L, NAT(min(L, 3)), 8)
    Y = torch.empty((len(r), (L + 1) ** 2), device="cuda")
    B.eqconv_spherical_harmonics(conv.plan, len(r), to_dev(r), Y)
    ref = sh(r.astype(np.float64), L)
    assert_close("Y", Y.cpu().numpy(), ref)


# ------------------------------------------------------------------ CSR

@pytest.mark.parametrize("N,E,pattern", [
    (1, 10, "random"), (7, 0, "random"), (300, 5000, "random"), (256, 40000, "sorted"),
    (70000, 200000, "random"),        # three radix passes
    (100, 9000, "one_hot"),           # every edge into one node
    (5000, 123457, "reversed"),
])
def test_csr_bit_exact(N, E, pattern):
    rng = np.random.default_rng(N + E)
    s = rng.integers(0, N, E).astype(np.int32)
    rcv = rng.integers(0, N, E).astype(np.int32)
    if pattern == "sorted":
        rcv = np.sort(rcv).astype(np.int32)
    elif pattern == "one_hot":
        rcv[:] = N // 2
    elif pattern == "reversed":
        rcv = np.sort(rcv)[::-1].copy().astype(np.int32)
    conv = EqConv("0e", 0, "0e", 4)
    g = conv.graph(to_dev(s) if E else torch.zeros(0, dtype=torch.int32, device="cuda"),
                   to_dev(rcv) if E else torch.zeros(0, dtype=torch.int32, device="cuda"), N)
    torch.cuda.synchronize()
    res = dict(recv_ptr=g.recv_ptr.cpu().numpy(), recv_perm=g.recv_perm[:E].cpu().numpy(),
               send_ptr=g.send_ptr.cpu().numpy(), send_perm=g.send_perm[:E].cpu().numpy())
    check_csr(res, s, rcv, N)


# ------------------------------------------------------------------ conv parity

CASES = [
    # (L_in, L_sh, L_out, C, N, E)
    (1, 2, 2, 32, 64, 1500),
    (2, 2, 2, 128, 300, 9000),
    (2, 2, 2, 132, 97, 4000),       # ragged channel tail, 2 tiles
    (2, 2, 2, 36, 50, 2000),
    (2, 2, 2, 4, 40, 800),
    (3, 3, 3, 128, 120, 5000),
    (3, 3, 3, 260, 40, 1300),
    (0, 1, 1, 64, 60, 900),
    (2, 0, 2, 16, 30, 500),
    (3, 2, 1, 8, 30, 600),
    (1, 3, 2, 128, 50, 1200),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "L%d%d%d_C%d" % c[:4])
@pytest.mark.parametrize("det", [True, False], ids=["det", "atomic"])
def test_conv_parity(case, det):
    L_in, L_sh, L_out, C, N, E = case
    s, rcv, r, x, w, gy = random_case(N, E, C, L_in, L_sh, L_out, seed=hash(case) % 1000)
    r[3] = 0.0  # a zero-length edge
    ins, outs = NAT(L_in), NAT(L_out)
    res = run_gpu(ins, L_sh, outs, C, N, s, rcv, r, x, w, gy, det=det)
    assert res["status"] == 0
    check_csr(res, s, rcv, N)
    check_all(res, oracle_full(ins, L_sh, outs, C, N, s, rcv, r, x, w, gy))


@pytest.mark.parametrize("lmax", [2, 3])
@pytest.mark.parametrize("vec", [(2, 2), (4, 4), (2, 4), (4, 2), (1, 1), (2, 1)])
def test_vector_widths_agree_with_oracle(vec, lmax):
    """Width 1 exists for plans with an l = 3 block and falls back to 2 else."""
    L_in, L_sh, L_out, C, N, E = lmax, lmax, lmax, 128, 120, 3000
    s, rcv, r, x, w, gy = random_case(N, E, C, L_in, L_sh, L_out, seed=5)
    ins = NAT(lmax)
    ref = oracle_full(ins, L_sh, ins, C, N, s, rcv, r, x, w, gy)
    for det in (True, False):
        check_all(run_gpu(ins, L_sh, ins, C, N, s, rcv, r, x, w, gy, det=det, vec=vec), ref)


@pytest.mark.parametrize("budget", [1, 150_000, 0])
def test_gather_bands_agree_with_oracle(budget):
    """Splitting the gathered node range into bands (budget 1 B: one band per
    node up to 64 bands; 150 kB: a few bands; 0: none) changes only the
    grouping of sums."""
    L_in, L_sh, L_out, C, N, E = 2, 2, 2, 132, 150, 5000
    s, rcv, r, x, w, gy = random_case(N, E, C, L_in, L_sh, L_out, seed=21)
    ins = NAT(2)
    ref = oracle_full(ins, L_sh, ins, C, N, s, rcv, r, x, w, gy)
    for vec in ((2, 2), (4, 4)):
        for det in (True, False):
            conv = EqConv(ins, L_sh, ins, C)
            conv.set_vec(*vec)
            conv.set_gather_budget(budget)
            g = conv.graph(to_dev(s), to_dev(rcv), N)
            xd, rd, wd = to_dev(x), to_dev(r), to_dev(w)
            y = conv.forward_raw(g, xd, rd, wd)
            dx, dw, dr = conv.backward_raw(g, xd, rd, wd, to_dev(gy), deterministic=det)
            torch.cuda.synchronize()
            assert B.eqconv_get_device_error(conv.plan) == B.EQCONV_OK
            check_all(dict(y=y.cpu().numpy(), dx=dx.cpu().numpy(), dw=dw.cpu().numpy(), dr=dr.cpu().numpy()), ref)


def test_bands_deterministic_mode_reproducible():
    L_in, L_sh, L_out, C, N, E = 2, 2, 2, 128, 300, 9000
    s, rcv, r, x, w, gy = random_case(N, E, C, L_in, L_sh, L_out, seed=22)
    ins = NAT(2)
    conv = EqConv(ins, L_sh, ins, C)
    conv.set_gather_budget(50_000)
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    xd, rd, wd, gd = to_dev(x), to_dev(r), to_dev(w), to_dev(gy)
    outs = []
    for _ in range(2):
        y = conv.forward_raw(g, xd, rd, wd)
        dx, dw, dr = conv.backward_raw(g, xd, rd, wd, gd, deterministic=True)
        torch.cuda.synchronize()
        outs.append([t.cpu().numpy().tobytes() for t in (y, dx, dw, dr)])
    assert outs[0] == outs[1]


def test_tiny_workload_full():
    """The 256-atom periodic box (C=32, 0e+1o -> 0e+1o+2e, L_sh=2), checked in full."""
    W = wl.WORKLOADS["tiny"]
    s, rcv, r = wl.make_graph(W)
    P = len(B.eqconv_enumerate_paths(W.irreps_in, W.L_sh, W.irreps_out))
    x = wl.features(W.N, 4, W.C, wl.SEED_X)
    w = wl.weights(len(s), P, W.C)
    gy = wl.features(W.N, 9, W.C, wl.SEED_GY)
    ref = oracle_full(W.irreps_in, W.L_sh, W.irreps_out, W.C, W.N, s, rcv, r, x, w, gy)
    for det in (True, False):
        res = run_gpu(W.irreps_in, W.L_sh, W.irreps_out, W.C, W.N, s, rcv, r, x, w, gy, det=det)
        check_csr(res, s, rcv, W.N)
        check_all(res, ref)


# ------------------------------------------------------------------ determinism

def test_deterministic_mode_is_bitwise_reproducible():
    L_in, L_sh, L_out, C, N, E = 2, 2, 2, 128, 400, 20000
    s, rcv, r, x, w, gy = random_case(N, E, C, L_in, L_sh, L_out, seed=11)
    ins = NAT(2)
    conv = EqConv(ins, L_sh, ins, C)
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    xd, rd, wd, gd = to_dev(x), to_dev(r), to_dev(w), to_dev(gy)
    outs = []
    for _ in range(3):
        y = conv.forward_raw(g, xd, rd, wd)
        dx, dw, dr = conv.backward_raw(g, xd, rd, wd, gd, deterministic=True)
        torch.cuda.synchronize()
        outs.append([t.cpu().numpy().tobytes() for t in (y, dx, dw, dr)])
    assert outs[0] == outs[1] == outs[2]


# ------------------------------------------------------------------ edge cases

def test_empty_graph_and_isolated_nodes():
    C, N = 16, 10
    ins = NAT(2)
    conv = EqConv(ins, 2, ins, C)
    e = torch.zeros(0, dtype=torch.int32, device="cuda")
    g = conv.graph(e, e, N)
    x = torch.randn(N, 9, C, device="cuda")
    r = torch.zeros(0, 3, device="cuda")
    w = torch.zeros(0, conv.P, C, device="cuda")
    y = conv.forward_raw(g, x, r, w)
    for det in (True, False):
        dx, dw, dr = conv.backward_raw(g, x, r, w, torch.randn_like(y), deterministic=det)
        assert torch.all(dx == 0)
    assert torch.all(y == 0)


def test_high_degree_receiver_and_duplicates():
    L_in, L_sh, L_out, C, N, E = 2, 2, 2, 64, 20, 3000
    s, rcv, r, x, w, gy = random_case(N, E, C, L_in, L_sh, L_out, seed=3)
    rcv[:2500] = 7          # one receiver with 2500 in-edges (many chunks)
    s[:100] = 3             # duplicated (3 -> 7) edges and a high out-degree sender
    s[100:110] = 7          # self-loops
    ins = NAT(2)
    ref = oracle_full(ins, L_sh, ins, C, N, s, rcv, r, x, w, gy)
    for det in (True, False):
        check_all(run_gpu(ins, L_sh, ins, C, N, s, rcv, r, x, w, gy, det=det), ref)


def test_out_of_range_sender_sets_status_without_fault():
    L_in, L_sh, L_out, C, N, E = 1, 1, 1, 8, 10, 50
    s, rcv, r, x, w, gy = random_case(N, E, C, L_in, L_sh, L_out, seed=4)
    s[5] = N + 3
    res = run_gpu(NAT(1), 1, NAT(1), C, N, s, rcv, r, x, w, gy, det=False)
    assert res["status"] == B.EQCONV_ERR_DEVICE_CHECK


def test_bad_arguments_are_rejected():
    conv = EqConv(NAT(1), 1, NAT(1), 8)
    e = torch.zeros(4, dtype=torch.int32, device="cuda")
    g = conv.graph(e, e, 2)
    x = torch.zeros(2, 4, 8, device="cuda")
    w = torch.zeros(4, conv.P, 8, device="cuda")
    r = torch.ones(4, 3, device="cuda")
    y = torch.zeros(2, 4, 8, device="cuda")
    with pytest.raises(B.EqconvError) as ei:
        B.eqconv_forward(conv.plan, g.c, x.data_ptr() + 4, r, w, y)   # misaligned
    assert ei.value.status == B.EQCONV_ERR_INVALID_ARG
    C2 = EqConv(NAT(2), 2, NAT(2), 512)
    assert B.eqconv_backward_workspace_bytes(C2.plan, 100) > 0
    with pytest.raises(B.EqconvError) as ei:
        g2 = C2.graph(e, e, 2)
        z = torch.zeros(2, 9, 512, device="cuda")
        ww = torch.zeros(4, C2.P, 512, device="cuda")
        B.eqconv_backward(C2.plan, g2.c, z, r, ww, z, z.clone(), ww.clone(), r.clone(), None, 0, 1)
    assert ei.value.status == B.EQCONV_ERR_WORKSPACE


# ------------------------------------------------------------------ autograd

def test_autograd_function_matches_raw_calls():
    L_in, L_sh, L_out, C, N, E = 2, 2, 2, 32, 40, 700
    s, rcv, r, x, w, gy = random_case(N, E, C, L_in, L_sh, L_out, seed=9)
    ins = NAT(2)
    conv = EqConv(ins, L_sh, ins, C)
    g = conv.graph(to_dev(s), to_dev(rcv), N)
    xd = to_dev(x).requires_grad_()
    rd = to_dev(r).requires_grad_()
    wd = to_dev(w).requires_grad_()
    y = conv(g, xd, rd, wd)
    (y * to_dev(gy)).sum().backward()
    ref = oracle_full(ins, L_sh, ins, C, N, s, rcv, r, x, w, gy)
    assert_close("y", y.detach().cpu().numpy(), ref[0])
    assert_close("dx", xd.grad.cpu().numpy(), ref[1])
    assert_close("dw", wd.grad.cpu().numpy(), ref[2])
    assert_close("dr", rd.grad.cpu().numpy(), ref[3])
