"""Shared pieces of the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

from equivariant_gnn_message_edge_b200.conv import EqConv
from oracle import conv as oconv
from oracle.csr import csr
from oracle.sh import sh
from tests.helpers import within_tol

REL, ABS = 1e-5, 1e-6


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def run_gpu(ins, L_sh, outs, C, N, senders, receivers, r, x, w, gy=None, det=True, vec=None, all_parity=False,
            per_path=False):
    conv = EqConv(ins, L_sh, outs, C, all_parity=all_parity, per_path=per_path)
    if vec is not None:
        conv.set_vec(*vec)
    s_d, r_d = to_dev(senders), to_dev(receivers)
    g = conv.graph(s_d, r_d, N)
    x_d, rv_d, w_d = to_dev(x), to_dev(r), to_dev(w)
    y = conv.forward_raw(g, x_d, rv_d, w_d)
    out = dict(y=y, recv_ptr=g.recv_ptr, recv_perm=g.recv_perm[:g.E], send_ptr=g.send_ptr,
               send_perm=g.send_perm[:g.E])
    if gy is not None:
        dx, dw, dr = conv.backward_raw(g, x_d, rv_d, w_d, to_dev(gy), deterministic=det)
        out.update(dx=dx, dw=dw, dr=dr)
    torch.cuda.synchronize()
    status = conv_status(conv)
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["status"] = status
    res["D_out"], res["path_rows"], res["paths"] = conv.D_out, conv.path_rows, conv.paths
    return res


def conv_status(conv):
    from equivariant_gnn_message_edge_b200 import binding as B
    return B.eqconv_get_device_error(conv.plan)


def oracle_full(ins, L_sh, outs, C, N, senders, receivers, r, x, w, gy=None, per_path=False):
    prob = oconv.Problem(ins, L_sh, outs, C, per_path=per_path)
    return oconv.full(prob, N, senders, receivers, r, x, w, gy)


def assert_close(name, got, ref):
    ok, err, bound = within_tol(got, ref, REL, ABS)
    assert ok, f"{name}: max|err| = {err:.3e} > bound {bound:.3e}"
    return err / max(bound, 1e-30)


def check_all(res, ref, with_bwd=True):
    assert_close("y", res["y"], ref[0] if with_bwd else ref)
    if with_bwd:
        _, dx, dw, dr = ref
        assert_close("dx", res["dx"], dx)
        assert_close("dw", res["dw"], dw)
        assert_close("dr", res["dr"], dr)


def check_csr(res, senders, receivers, N):
    rp, rperm = csr(receivers, N)
    sp, sperm = csr(senders, N)
    assert np.array_equal(res["recv_ptr"], rp)
    assert np.array_equal(res["recv_perm"], rperm)
    assert np.array_equal(res["send_ptr"], sp)
    assert np.array_equal(res["send_perm"], sperm)


__all__ = ["run_gpu", "oracle_full", "assert_close", "check_all", "check_csr", "to_dev", "sh", "oconv", "csr"]
