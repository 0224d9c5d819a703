"""The equivariant message-passing convolution, forward and backward (oracle).

Test infrastructure only (see ``oracle/__init__.py``).

Definition (e3j, abstract / Table 1; FlashCart App. B, §4 and App. D):

    y[i,l3,m3,c] = sum_{e: recv(e)=i} sum_{p=(l1,l2,l3)} w[e,p,c]
                   sum_{m1,m2} C_p[m1,m2,m3] x[send(e),l1,m1,c] Y_{l2 m2}(r_e / |r_e|)

with C_p the real CG of ``oracle/cg.py`` and Y the component-normalised real
harmonics of ``oracle/sh.py``.  Backward given gy (FlashCart §2: forces are
energy gradients; App. C/D: gradients for both inputs and the weight):

    dx[j,l1,m1,c] = sum_{e: send(e)=j} sum_p w[e,p,c] sum_{m2,m3} C_p Y_{l2m2} gy[recv(e),l3,m3,c]
    dw[e,p,c]     = sum_{m1,m2,m3} C_p x[send(e),l1,m1,c] Y_{l2m2} gy[recv(e),l3,m3,c]
    gY[e,l2,m2]   = sum_c sum_{p with l2} w[e,p,c] sum_{m1,m3} C_p x gy
    dr[e]         = (dY/dr_e)^T gY[e]

Per-path retention (FlashCart App. D: the channel-diagonal product may keep
each path's output or sum the paths that land on the same irrep): with
``per_path=True`` every path writes its own output block, in path order, so
y[i, o3(p)+m3, c] holds path p alone and D_out = sum_p (2 l3 + 1); summing
the blocks of each output irrep gives the summed layout back.

Readings where the pages are silent: no 1/sqrt(P), fan-in or 1/avg-degree
factor inside the op (the weights carry all scaling); zero-length edges have
Y_0 = 1, Y_{l>0} = 0 and dr = 0; isolated receivers give y = 0.

Two independent implementations:
* ``forward_bruteforce`` / ``backward_bruteforce``: NumPy, per-edge messages
  materialised (the e3nn-jax style that Table 1 of the e3j page says overflows
  memory at scale) - small inputs only;
* ``forward`` / ``backward_*``: the plain C loops of ``conv_ref.c`` (fp64
  accumulation, OpenMP over output rows), for large inputs and row samples.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

import numpy as np

from . import build as _build
from .cg import real_cg
from .irreps import block_offsets, enumerate_paths, parse_irreps
from .sh import sh, sh_grad


@dataclass
class Problem:
    irreps_in: str
    L_sh: int
    irreps_out: str
    C: int
    per_path: bool = False
    paths: list = field(init=False)
    D_in: int = field(init=False)
    D_sh: int = field(init=False)
    D_out: int = field(init=False)
    layout_out: str = field(init=False)

    def __post_init__(self):
        ins, outs = parse_irreps(self.irreps_in), parse_irreps(self.irreps_out)
        self.paths = enumerate_paths(ins, self.L_sh, outs)
        self.D_in = block_offsets(ins)[1]
        self.D_sh = (self.L_sh + 1) ** 2
        if self.per_path:
            # one block per path, in path order
            off, names = 0, []
            for q in self.paths:
                q["off3"] = off
                off += 2 * q["l3"] + 1
                names.append(f"{q['l3']}{'e' if outs[q['i3']][1] > 0 else 'o'}")
            self.D_out = off
            self.layout_out = "+".join(names)
        else:
            self.D_out = block_offsets(outs)[1]
            self.layout_out = self.irreps_out

    @property
    def P(self) -> int:
        return len(self.paths)

    def cg(self, p: int) -> np.ndarray:
        q = self.paths[p]
        return real_cg(q["l1"], q["l2"], q["l3"])

    def c_tables(self):
        """(pd int32[6P], cgo int64[P], cg float64[...]) for conv_ref.c."""
        pd, cgo, blocks, off = [], [], [], 0
        for p, q in enumerate(self.paths):
            d1, d2, d3 = 2 * q["l1"] + 1, 2 * q["l2"] + 1, 2 * q["l3"] + 1
            pd += [q["off1"], d1, q["off2"], d2, q["off3"], d3]
            cgo.append(off)
            blocks.append(np.ascontiguousarray(self.cg(p), dtype=np.float64).reshape(-1))
            off += d1 * d2 * d3
        return (np.asarray(pd, dtype=np.int32), np.asarray(cgo, dtype=np.int64),
                np.concatenate(blocks) if blocks else np.zeros(0))


# --------------------------------------------------------------------------
# NumPy brute force: materialise every per-edge message
# --------------------------------------------------------------------------

def edge_messages(prob: Problem, senders, r, x, w) -> np.ndarray:
    """msg[e, o3+m3, c] for every edge (fp64)."""
    Y = sh(r, prob.L_sh)
    E = len(senders)
    msg = np.zeros((E, prob.D_out, prob.C))
    xs = np.asarray(x, dtype=np.float64)[senders]
    w = np.asarray(w, dtype=np.float64)
    for p, q in enumerate(prob.paths):
        d1, d2, d3 = 2 * q["l1"] + 1, 2 * q["l2"] + 1, 2 * q["l3"] + 1
        Cp = prob.cg(p)
        xb = xs[:, q["off1"]:q["off1"] + d1, :]
        Yb = Y[:, q["off2"]:q["off2"] + d2]
        t = np.einsum("abk,eb,eac->ekc", Cp, Yb, xb)
        msg[:, q["off3"]:q["off3"] + d3, :] += w[:, p, None, :] * t
    return msg


def forward_bruteforce(prob: Problem, N: int, senders, receivers, r, x, w) -> np.ndarray:
    msg = edge_messages(prob, senders, r, x, w)
    y = np.zeros((N, prob.D_out, prob.C))
    np.add.at(y, np.asarray(receivers), msg)
    return y


def backward_bruteforce(prob: Problem, N: int, senders, receivers, r, x, w, gy):
    """(dx, dw, dr) by per-edge materialisation (fp64)."""
    Y = sh(r, prob.L_sh)
    J = sh_grad(r, prob.L_sh)
    E = len(senders)
    xs = np.asarray(x, dtype=np.float64)[senders]
    gyr = np.asarray(gy, dtype=np.float64)[receivers]
    w = np.asarray(w, dtype=np.float64)
    dx_e = np.zeros((E, prob.D_in, prob.C))
    dw = np.zeros((E, prob.P, prob.C))
    gY = np.zeros((E, prob.D_sh))
    for p, q in enumerate(prob.paths):
        d1, d2, d3 = 2 * q["l1"] + 1, 2 * q["l2"] + 1, 2 * q["l3"] + 1
        Cp = prob.cg(p)
        xb = xs[:, q["off1"]:q["off1"] + d1, :]
        gb = gyr[:, q["off3"]:q["off3"] + d3, :]
        Yb = Y[:, q["off2"]:q["off2"] + d2]
        dx_e[:, q["off1"]:q["off1"] + d1, :] += w[:, p, None, :] * np.einsum("abk,eb,ekc->eac", Cp, Yb, gb)
        G = np.einsum("abk,eac,ekc->ebc", Cp, xb, gb)          # [E, d2, C]
        dw[:, p, :] = np.einsum("ebc,eb->ec", G, Yb)
        gY[:, q["off2"]:q["off2"] + d2] += np.einsum("ebc,ec->eb", G, w[:, p, :])
    dx = np.zeros((N, prob.D_in, prob.C))
    np.add.at(dx, np.asarray(senders), dx_e)
    dr = np.einsum("ekj,ek->ej", J, gY)
    return dx, dw, dr


# --------------------------------------------------------------------------
# C loops (conv_ref.c)
# --------------------------------------------------------------------------

def _p(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _c32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def max_threads() -> int:
    return int(_build.load().oracle_max_threads())


def forward(prob: Problem, recv_ptr, recv_perm, senders, Y, x, w, rows=None, nthreads=0):
    """y rows (fp64) for the receivers in ``rows`` (all when None).  Y is the
    fp64 harmonics table [E, D_sh] from ``oracle.sh.sh``."""
    lib = _build.load()
    N = len(recv_ptr) - 1
    rows = np.arange(N, dtype=np.int32) if rows is None else _c32(rows)
    pd, cgo, cg = prob.c_tables()
    Y = np.ascontiguousarray(Y, dtype=np.float64)
    out = np.zeros((len(rows), prob.D_out, prob.C))
    recv_ptr, recv_perm, senders, x, w = _c32(recv_ptr), _c32(recv_perm), _c32(senders), _f32(x), _f32(w)
    lib.oracle_forward(ctypes.c_int(prob.C), ctypes.c_int(prob.D_in), ctypes.c_int(prob.D_sh),
                       ctypes.c_int(prob.D_out), ctypes.c_int(prob.P), _p(pd, ctypes.c_int),
                       _p(cgo, ctypes.c_int64), _p(cg, ctypes.c_double), ctypes.c_int(len(rows)),
                       _p(rows, ctypes.c_int), _p(recv_ptr, ctypes.c_int), _p(recv_perm, ctypes.c_int),
                       _p(senders, ctypes.c_int), _p(x, ctypes.c_float), _p(Y, ctypes.c_double),
                       _p(w, ctypes.c_float), _p(out, ctypes.c_double), ctypes.c_int(nthreads))
    return out


def backward_dx(prob: Problem, send_ptr, send_perm, receivers, Y, gy, w, rows=None, nthreads=0):
    lib = _build.load()
    N = len(send_ptr) - 1
    rows = np.arange(N, dtype=np.int32) if rows is None else _c32(rows)
    pd, cgo, cg = prob.c_tables()
    Y = np.ascontiguousarray(Y, dtype=np.float64)
    out = np.zeros((len(rows), prob.D_in, prob.C))
    send_ptr, send_perm, receivers, gy, w = _c32(send_ptr), _c32(send_perm), _c32(receivers), _f32(gy), _f32(w)
    lib.oracle_backward_dx(ctypes.c_int(prob.C), ctypes.c_int(prob.D_in), ctypes.c_int(prob.D_sh),
                           ctypes.c_int(prob.D_out), ctypes.c_int(prob.P), _p(pd, ctypes.c_int),
                           _p(cgo, ctypes.c_int64), _p(cg, ctypes.c_double), ctypes.c_int(len(rows)),
                           _p(rows, ctypes.c_int), _p(send_ptr, ctypes.c_int), _p(send_perm, ctypes.c_int),
                           _p(receivers, ctypes.c_int), _p(gy, ctypes.c_float), _p(Y, ctypes.c_double),
                           _p(w, ctypes.c_float), _p(out, ctypes.c_double), ctypes.c_int(nthreads))
    return out


def backward_edges(prob: Problem, senders, receivers, Y, x, gy, w, edges=None, nthreads=0):
    """(dw rows [n, P, C], gY rows [n, D_sh]) for the listed edges (fp64)."""
    lib = _build.load()
    E = len(senders)
    edges = np.arange(E, dtype=np.int32) if edges is None else _c32(edges)
    pd, cgo, cg = prob.c_tables()
    Y = np.ascontiguousarray(Y, dtype=np.float64)
    dw = np.zeros((len(edges), prob.P, prob.C))
    gY = np.zeros((len(edges), prob.D_sh))
    senders, receivers, x, gy, w = _c32(senders), _c32(receivers), _f32(x), _f32(gy), _f32(w)
    lib.oracle_backward_edges(ctypes.c_int(prob.C), ctypes.c_int(prob.D_in), ctypes.c_int(prob.D_sh),
                              ctypes.c_int(prob.D_out), ctypes.c_int(prob.P), _p(pd, ctypes.c_int),
                              _p(cgo, ctypes.c_int64), _p(cg, ctypes.c_double), ctypes.c_int(len(edges)),
                              _p(edges, ctypes.c_int), _p(senders, ctypes.c_int), _p(receivers, ctypes.c_int),
                              _p(x, ctypes.c_float), _p(gy, ctypes.c_float), _p(Y, ctypes.c_double),
                              _p(w, ctypes.c_float), _p(dw, ctypes.c_double), _p(gY, ctypes.c_double),
                              ctypes.c_int(nthreads))
    return dw, gY


def dr_from_gY(r, gY, L_sh: int) -> np.ndarray:
    """dr[e] = (dY/dr_e)^T gY[e]."""
    return np.einsum("ekj,ek->ej", sh_grad(r, L_sh), gY)


def full(prob: Problem, N: int, senders, receivers, r, x, w, gy=None, nthreads=0):
    """Whole forward (and backward when gy is given) through the C loops."""
    from .csr import csr
    rp, rperm = csr(receivers, N)
    sp, sperm = csr(senders, N)
    Y = sh(r, prob.L_sh)
    y = forward(prob, rp, rperm, senders, Y, x, w, nthreads=nthreads)
    if gy is None:
        return y
    dx = backward_dx(prob, sp, sperm, receivers, Y, gy, w, nthreads=nthreads)
    dw, gY = backward_edges(prob, senders, receivers, Y, x, gy, w, nthreads=nthreads)
    dr = dr_from_gY(r, gY, prob.L_sh)
    return y, dx, dw, dr
