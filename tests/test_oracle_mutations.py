"""Planted mistakes: each plausible error in the oracle must fail a pin.

The mistakes are planted in the oracle, on the CPU, through monkeypatching;
each test checks that one of the pins of test_oracle_*.py sees it.  This is
what makes the pins trustworthy: a dropped term, a wrong sign or index, or a
transposed operand does not pass silently.
"""
import numpy as np

from oracle import cg as cgmod
from oracle import conv
from oracle import sh as shmod
from tests.helpers import block_wigner, random_rotation, small_problem
from tests.test_oracle_sh import closed_forms


def _equivariance_error(prob, N, s, rcv, r, x, w):
    R = random_rotation(11)
    Din, Dout = block_wigner(R, prob.irreps_in), block_wigner(R, prob.irreps_out)
    y = conv.forward_bruteforce(prob, N, s, rcv, r, x, w)
    y_rot = conv.forward_bruteforce(prob, N, s, rcv, r.astype(np.float64) @ R.T,
                                    np.einsum("ab,nbc->nac", Din, x.astype(np.float64)), w)
    return np.max(np.abs(y_rot - np.einsum("ab,nbc->nac", Dout, y))) / np.max(np.abs(y))


def test_sign_error_in_sh_fails_closed_forms(monkeypatch):
    real = shmod.sh

    def bad(r, L):
        Y = real(r, L)
        Y[..., 5] = -Y[..., 5]             # flip Y_{2,-1}
        return Y
    u = np.random.default_rng(0).standard_normal((20, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    assert np.max(np.abs(real(u, 3) - closed_forms(u))) < 1e-12
    assert np.max(np.abs(bad(u, 3) - closed_forms(u))) > 1e-3


def test_reversed_m2_in_one_cg_fails_equivariance(monkeypatch):
    N = 8
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=30, C=3)
    assert _equivariance_error(prob, N, s, rcv, r, x, w) < 1e-10
    real = cgmod.real_cg

    def bad(l1, l2, l3):
        C = real(l1, l2, l3)
        return C[:, ::-1, :].copy() if (l1, l2, l3) == (1, 2, 1) else C
    monkeypatch.setattr(conv, "real_cg", bad)
    assert _equivariance_error(prob, N, s, rcv, r, x, w) > 1e-3


def test_transposition_mistakes_are_harmless_or_shape_errors():
    """m1 <-> m3 transposition: for l1 != l3 the shapes differ (the mistake
    cannot run); for every natural-parity path with l1 = l3 the coupling is
    symmetric in m1 <-> m3, so the transposed tensor gives the same result.
    Odd paths (both-parity variant) are antisymmetric there."""
    import itertools
    for l1, l2 in itertools.product(range(4), repeat=2):
        for l3 in [l1]:
            if abs(l1 - l2) <= l3 <= l1 + l2:
                C = cgmod.real_cg(l1, l2, l3)
                sign = 1 if (l1 + l2 + l3) % 2 == 0 else -1
                assert np.max(np.abs(C - sign * C.transpose(2, 1, 0))) < 1e-13


def test_dropped_path_in_forward_fails_bilinearity(monkeypatch):
    N = 9
    prob, s, rcv, r, x, w, gy = small_problem(N=N, E=40, C=4)
    y, dx, dw, dr = conv.full(prob, N, s, rcv, r, x, w, gy)
    w_dropped = w.copy()
    w_dropped[:, 4, :] = 0.0               # forward silently skips path 4
    y_bad = conv.full(prob, N, s, rcv, r, x, w_dropped)
    a, b = float((gy * y_bad).sum()), float((w * dw).sum())
    assert abs(a - b) > 1e-6 * abs(b)


def test_missing_radial_projection_fails_finite_differences(monkeypatch):
    rng = np.random.default_rng(2)
    r = rng.standard_normal((10, 3)) * 2.0
    g = shmod.sh_grad(r, 2)
    u = r / np.linalg.norm(r, axis=1, keepdims=True)
    radial = np.einsum("ekj,ej->ek", g, u)
    assert np.max(np.abs(radial)) < 1e-12
    # a gradient that forgot the projection (grad f(u) / |r| only) differs
    # from finite differences in the radial direction:
    h = 1e-6
    fd_radial = (shmod.sh(r + h * u, 2) - shmod.sh(r - h * u, 2)) / (2 * h)
    assert np.max(np.abs(fd_radial)) < 1e-8


def _dbl_fd_failures(dbl_fn):
    """Names of the inputs whose central-difference pin (test_oracle_dbl.py)
    a double-backward implementation fails."""
    from tests.test_oracle_dbl import CASES, _S, _setup
    prob, s, rcv, r, x, w, gy, a, b, q = _setup(CASES[1], seed=3)
    grads = dbl_fn(prob, 8, s, rcv, r, x, w, gy, a, b, q)
    rng = np.random.default_rng(11)
    h, fails, args = 1e-6, [], dict(r=r, x=x, w=w, gy=gy)
    for name, g in zip(("x", "w", "gy", "r"), grads):
        d = rng.standard_normal(args[name].shape)
        p, m = dict(args), dict(args)
        p[name] = args[name] + h * d
        m[name] = args[name] - h * d
        fd = (_S(prob, 8, s, rcv, p["r"], p["x"], p["w"], p["gy"], a, b, q)[0] -
              _S(prob, 8, s, rcv, m["r"], m["x"], m["w"], m["gy"], a, b, q)[0]) / (2 * h)
        an = float((g * d).sum())
        if abs(fd - an) >= 1e-6 * max(1.0, abs(an)):
            fails.append(name)
    return fails


def test_double_backward_mistakes_fail_the_difference_pins():
    """A dropped Hessian term, the wrong cotangent in gY, a dropped rho term
    and a flipped sign each fail the central-difference pin of one input."""
    import inspect
    from oracle import dbl
    src = inspect.getsource(dbl)
    assert _dbl_fd_failures(dbl.double_backward_bruteforce) == []
    mistakes = {
        "r": ('+ np.einsum("ekij,ek,ej->ei", H, gY1, q)', ""),
        "r ": ('np.einsum("ebc,ec->eb", Gx, b[:, p])', 'np.einsum("ebc,ec->eb", Ga, b[:, p])'),
        "gy": ("+ wp * msg(Rb, xb)", ""),
        "x": ("g_x_e[:, o1:o1 + d1, :] += bp * uY + wp * uR", "g_x_e[:, o1:o1 + d1, :] += bp * uY - wp * uR"),
    }
    for expect, (good, bad) in mistakes.items():
        assert good in src
        ns = {}
        code = src.replace(good, bad).replace("from .conv import", "from oracle.conv import")
        exec(compile(code.replace("from .sh import", "from oracle.sh import"), "planted", "exec"), ns)
        assert expect.strip() in _dbl_fd_failures(ns["double_backward_bruteforce"])


def test_variant_mistakes_fail_the_variant_pins():
    """Both-parity and per-path outputs: taking the real part for an odd
    path (which is zero, so the pseudo-tensor block vanishes), or swapping
    the output blocks of two paths of opposite parity, each fail a pin of
    test_oracle_modes.py (the cross product; the inversion signs)."""
    from equivariant_gnn_message_edge_b200.workloads import both_parity_irreps, natural_irreps
    # (1) odd coupling taken as the real part: the cross-product pin fails
    real = cgmod._real_cg_cached.__wrapped__

    def real_part(l1, l2, l3):
        C = real(l1, l2, l3)
        return np.zeros_like(C) if (l1 + l2 + l3) % 2 else C
    C_bad = real_part(1, 1, 1)
    u, v = np.array([0.3, -1.0, 0.4]), np.array([1.1, 0.2, -0.7])
    perm = [1, 2, 0]
    want = np.cross(u, v)[perm] / np.sqrt(2.0)
    assert np.max(np.abs(np.abs(np.einsum("abk,a,b->k", C_bad, u[perm], v[perm])) - np.abs(want))) > 1e-3
    # (2) two per-path blocks of the same size but opposite parity swapped
    # ((1,1,2) -> 2e and (2,1,2) -> 2o): the inversion-sign pin fails
    from tests.helpers import parity_signs
    N = 6
    pp = conv.Problem(natural_irreps(2), 2, both_parity_irreps(2), 3, per_path=True)
    rng = np.random.default_rng(1)
    s = rng.integers(0, N, 30).astype(np.int32)
    rcv = rng.integers(0, N, 30).astype(np.int32)
    r = rng.standard_normal((30, 3))
    x = rng.standard_normal((N, pp.D_in, 3))
    w = rng.standard_normal((30, pp.P, 3))
    pin, pout = parity_signs(pp.irreps_in), parity_signs(pp.layout_out)

    def parity_error():
        y = conv.forward_bruteforce(pp, N, s, rcv, r, x, w)
        y_inv = conv.forward_bruteforce(pp, N, s, rcv, -r, pin[None, :, None] * x, w)
        return np.max(np.abs(y_inv - pout[None, :, None] * y)) / np.max(np.abs(y))
    assert parity_error() < 1e-12
    a = next(k for k, q in enumerate(pp.paths) if (q["l1"], q["l2"], q["l3"]) == (1, 1, 2))
    b = next(k for k, q in enumerate(pp.paths) if (q["l1"], q["l2"], q["l3"]) == (2, 1, 2))
    qa, qb = pp.paths[a], pp.paths[b]
    qa["off3"], qb["off3"] = qb["off3"], qa["off3"]
    try:
        assert parity_error() > 1e-3
    finally:
        qa["off3"], qb["off3"] = qb["off3"], qa["off3"]


def test_node_product_mistakes_fail_the_derivative_pin():
    """In the node-local product's backward, a flipped sign in dv or a
    dropped weight in du fails the exact directional-derivative pin."""
    import inspect
    from oracle import nodeprod
    from tests.test_oracle_nodeprod import _setup
    src = inspect.getsource(nodeprod)
    prob, u, v, w, gy = _setup(2, 2, 2, seed=6)

    def fails(mod_src):
        ns = {}
        exec(compile(mod_src.replace("from .conv import", "from oracle.conv import"), "planted", "exec"), ns)
        du, dv, dw = ns["node_product_backward"](prob, u, v, w, gy)
        S = lambda uu, vv, ww: float((gy * nodeprod.node_product(prob, uu, vv, ww)).sum())
        s0 = S(u, v, w)
        rng = np.random.default_rng(3)
        bad = []
        for name, g in (("u", du), ("v", dv), ("w", dw)):
            d = rng.standard_normal(g.shape)
            args = dict(u=u, v=v, w=w)
            args[name] = args[name] + d
            if abs(S(args["u"], args["v"], args["w"]) - s0 - (g * d).sum()) > 1e-8 * max(1.0, abs(s0)):
                bad.append(name)
        return bad
    assert fails(src) == []
    good = 'dv[:, q["off2"]:q["off2"] + d2, :] += w[p] * '
    assert good in src
    assert "v" in fails(src.replace(good, 'dv[:, q["off2"]:q["off2"] + d2, :] -= w[p] * '))
    good = 'du[:, q["off1"]:q["off1"] + d1, :] += w[p] * '
    assert good in src
    assert "u" in fails(src.replace(good, 'du[:, q["off1"]:q["off1"] + d1, :] += '))


def test_radial_mistakes_fail_the_radial_pins():
    """In the radial weights' VJP, a dropped envelope-derivative term or a
    missing SiLU derivative fails the central-difference / autograd pins."""
    import inspect
    from oracle import radial
    from tests.test_oracle_radial import RC, _params
    src = inspect.getsource(radial)
    P, C = 2, 3
    params = _params(P, C, seed=4)
    rng = np.random.default_rng(5)
    d = rng.uniform(0.5, 4.9, 20)
    gw = rng.standard_normal((20, P, C))

    def err(mod_src):
        ns = {}
        exec(compile(mod_src, "planted", "exec"), ns)
        g_d, _ = ns["radial_weights_vjp"](d, RC, params, gw)
        h = 1e-6
        fd = ((radial.radial_weights(d + h, RC, params, P, C) - radial.radial_weights(d - h, RC, params, P, C)) *
              gw).sum((1, 2)) / (2 * h)
        return np.max(np.abs(fd - g_d)) / max(1.0, np.max(np.abs(fd)))
    assert err(src) < 1e-6
    good = " + g_u * envelope_grad(d, rc, p)"
    assert good in src and err(src.replace(good, "")) > 1e-3
    good = "g_z2 = (g_z3 @ W3.T) * _silu_grad(z2)"
    assert good in src and err(src.replace(good, "g_z2 = (g_z3 @ W3.T)")) > 1e-3
