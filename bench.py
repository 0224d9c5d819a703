#!/usr/bin/env python
"""Benchmark of the equivariant message-passing convolution hot path on B200.

One step = the whole path over one batch of synthetic input: edge layout
(receiver and sender CSR + stable permutations), fused forward, fused
deterministic backward (dx, dw, dr).  Default workload: the lmax=2 setting of
the e3j page's Table 1 (N=32768 nodes, C=128 channels, Poisson(45) in-degree,
irreps 0e+1o+2e, L_sh=2; E ~ 1.47M edges, 11 paths, w = 8.3 GB).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Throughput is unique bytes (every tensor the step reads or writes, counted
once) per second, and edges per second.  Multi-GPU runs are independent
replicas (the convolution needs no collective); the timed region is bracketed
by a barrier and a device synchronize, and the time is the max over ranks.
``--impl reference`` times the CPU oracle (fp64 C loops) on a bounded sample of
the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from equivariant_gnn_message_edge_b200 import workloads as wl  # noqa: E402

METRIC = "conv fwd / fwd+bwd GB/s and edges/s at lmax=2 C=128; % of B200 HBM peak"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------- sizes

def tensor_bytes(N, E, C, D_in, D_out, P):
    f = 4
    return dict(
        senders=4 * E, receivers=4 * E, recv_ptr=4 * (N + 1), recv_perm=4 * E, send_ptr=4 * (N + 1),
        send_perm=4 * E, x=f * N * D_in * C, r=f * E * 3, w=f * E * P * C, gy=f * N * D_out * C,
        y=f * N * D_out * C, dx=f * N * D_in * C, dw=f * E * P * C, dr=f * E * 3)


def byte_counts(N, E, C, D_in, D_out, P):
    t = tensor_bytes(N, E, C, D_in, D_out, P)
    fwd = sum(t[k] for k in ("x", "r", "w", "recv_ptr", "recv_perm", "senders", "y"))
    bwd = sum(t[k] for k in ("x", "r", "w", "gy", "send_ptr", "send_perm", "receivers", "dx", "dw", "dr"))
    graph = sum(t[k] for k in ("senders", "receivers", "recv_ptr", "recv_perm", "send_ptr", "send_perm"))
    # the step's unique bytes: every tensor the step reads or writes counted
    # once over the whole step (graph build + forward + backward) - the
    # headline; `kernels` counts each kernel's own tensors (the roofline's)
    step = sum(t.values())
    h2d = sum(t[k] for k in ("senders", "receivers", "x", "r", "w", "gy"))
    d2h = sum(t[k] for k in ("y", "dx", "dw", "dr"))
    return dict(fwd=fwd, bwd=bwd, graph=graph, step=step, h2d=h2d, d2h=d2h, kernels=graph + fwd + bwd)


FP32_PEAK_SM_MHZ = 1965.0     # clocks.max.sm of the B200s this runs on


def fp32_peak_tflops(sm_mhz=FP32_PEAK_SM_MHZ):
    """FP32 FMA peak: 148 SMs x 128 FMA lanes x 2 flop x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def fma_counts(paths, cg_table):
    """FMA per (edge, channel) of the forward and of the backward's h-form
    contraction as the kernels issue them, counted from the real CG tables
    (zero coefficients are skipped at compile time).  cg_table(l1, l2, l3)
    gives the [2l1+1][2l2+1][2l3+1] table."""
    fwd = bwd = 0
    for l1, l2, l3 in paths:
        d1, d2, d3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
        if l2 == 0:
            fwd += d1
            bwd += 2 * d1                      # dw = x . g, dx += w g
            continue
        fwd += d1 * d3 + min(d1, d3)           # A x (d3 x d1), then the weight
        t = np.asarray(cg_table(l1, l2, l3))
        nz = np.abs(t) > 0
        rows = int(nz.any(axis=2).sum())       # (m1, m2) rows with a nonzero coefficient
        bwd += int(nz.sum()) + 2 * rows + 2 * d1 + d2
    return fwd, bwd


def time_node_product(W, Nn, dev, stream, reps, reduce=lambda t: t):
    """Median device time and GB/s of the node-local product (forward, and
    backward with dw) on Nn nodes; bytes = each tensor read or written once
    per kernel (u, v, w, y; u, v, w, gy, du, dv, dw partials, dw)."""
    import torch

    from equivariant_gnn_message_edge_b200 import binding as B
    from equivariant_gnn_message_edge_b200.conv import NodeProduct
    op = NodeProduct(W.irreps_in, W.L_sh, W.irreps_out, W.C, per_path=W.per_path)
    gen = torch.Generator(device=dev).manual_seed(wl.SEED_X + 7)
    C, P = W.C, op.P
    with torch.cuda.stream(stream):
        u = torch.randn((Nn, op.D_u, C), generator=gen, device=dev)
        v = torch.randn((Nn, op.D_v, C), generator=gen, device=dev)
        w = torch.randn((P, C), generator=gen, device=dev)
        gy = torch.randn((Nn, op.D_out, C), generator=gen, device=dev)
        y = torch.empty_like(gy)
        du, dv, dw = torch.empty_like(u), torch.empty_like(v), torch.empty_like(w)
        nws = B.eqconv_node_product_workspace_bytes(op.plan, Nn)
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
    h = stream.cuda_stream
    fe, be = [], []
    for _ in range(reps + 1):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        B.eqconv_node_product(op.plan, Nn, u, v, w, y, h)
        ev[1].record(stream)
        B.eqconv_node_product_backward(op.plan, Nn, u, v, w, gy, du, dv, dw, ws, nws, h)
        ev[2].record(stream)
        fe.append(ev)
    stream.synchronize()
    f_ms = reduce(statistics.median([e[0].elapsed_time(e[1]) for e in fe[1:]]))     # max over ranks
    b_ms = reduce(statistics.median([e[1].elapsed_time(e[2]) for e in fe[1:]]))
    row = 4 * C * Nn
    fb = row * (op.D_u + op.D_v + op.D_out) + 4 * P * C
    bb = row * (2 * op.D_u + 2 * op.D_v + op.D_out) + 4 * P * C + 2 * nws + 4 * P * C
    peak = measured_peak()[0]
    return {"nodes": Nn, "paths": P, "fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4),
            "fwd_gbps": round(fb / (f_ms * 1e-3) / 1e9, 1), "bwd_gbps": round(bb / (b_ms * 1e-3) / 1e9, 1),
            "fwd_frac_of_measured_hbm": round(fb / (f_ms * 1e-3) / 1e9 / peak, 4),
            "bwd_frac_of_measured_hbm": round(bb / (b_ms * 1e-3) / 1e9 / peak, 4),
            "bytes": "fwd: u, v, w read, y written; bwd: u, v, w, gy read, du, dv written, dw partials written "
                     "and read, dw written"}


def time_symmetric_contraction(W, Nn, dev, stream, reps, reduce=lambda t: t, n_species=4):
    """Median device time and GB/s of the symmetric contraction of correlation
    order 2 (A (x) A with per-species weights; irreps of the workload's
    features in and out) on Nn nodes, forward and backward; bytes = each
    tensor read or written once per kernel (A, species, W1, W2, B; A,
    species, W1, W2, gB, dA, the weight-gradient partials written and read,
    dW1, dW2)."""
    import torch

    from equivariant_gnn_message_edge_b200 import binding as B
    from equivariant_gnn_message_edge_b200.conv import SymmetricContraction
    op = SymmetricContraction(W.irreps_in, W.irreps_out, W.C, n_species)
    gen = torch.Generator(device=dev).manual_seed(wl.SEED_X + 11)
    C, P, S = W.C, op.P, n_species
    with torch.cuda.stream(stream):
        A = torch.randn((Nn, op.D_A, C), generator=gen, device=dev)
        z = torch.randint(0, S, (Nn,), generator=gen, device=dev, dtype=torch.int32)
        W1 = torch.randn((S, op.L1N, C), generator=gen, device=dev)
        W2 = torch.randn((S, P, C), generator=gen, device=dev)
        gB = torch.randn((Nn, op.D_out, C), generator=gen, device=dev)
        out = torch.empty_like(gB)
        dA, dW1, dW2 = torch.empty_like(A), torch.empty_like(W1), torch.empty_like(W2)
        nws = B.eqconv_symmetric_contraction_workspace_bytes(op.plan, Nn)
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
    h = stream.cuda_stream
    fe = []
    for _ in range(reps + 1):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        B.eqconv_symmetric_contraction(op.plan, Nn, A, z, W1, W2, out, h)
        ev[1].record(stream)
        B.eqconv_symmetric_contraction_backward(op.plan, Nn, A, z, W1, W2, gB, dA, dW1, dW2, ws, nws, h)
        ev[2].record(stream)
        fe.append(ev)
    stream.synchronize()
    assert B.eqconv_get_device_error(op.plan, h) == B.EQCONV_OK
    f_ms = reduce(statistics.median([e[0].elapsed_time(e[1]) for e in fe[1:]]))     # max over ranks
    b_ms = reduce(statistics.median([e[1].elapsed_time(e[2]) for e in fe[1:]]))
    row = 4 * C * Nn
    wbytes = 4 * S * (op.L1N + P) * C
    fb = row * (op.D_A + op.D_out) + 4 * Nn + wbytes
    bb = row * (2 * op.D_A + op.D_out) + 4 * Nn + 2 * wbytes + 2 * nws
    peak = measured_peak()[0]
    return {"nodes": Nn, "species": S, "paths": P, "fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4),
            "fwd_gbps": round(fb / (f_ms * 1e-3) / 1e9, 1), "bwd_gbps": round(bb / (b_ms * 1e-3) / 1e9, 1),
            "fwd_frac_of_measured_hbm": round(fb / (f_ms * 1e-3) / 1e9 / peak, 4),
            "bwd_frac_of_measured_hbm": round(bb / (b_ms * 1e-3) / 1e9 / peak, 4),
            "bytes": "fwd: A, species, W1, W2 read, B written; bwd: A, species, W1, W2, gB read, dA written, "
                     "weight-gradient partials written and read, dW1, dW2 written"}


def device_inputs(W, D_in, D_out, P, dev, seed_offset=0):
    """Graph of workload W from the seeded NumPy generators; features, weights
    and output gradients drawn on the device by a seeded torch generator with
    the stated laws (x, gy ~ N(0, 1), w ~ N(0, 1/P)), which is much faster
    than drawing several GB on the host.  Returns (s, rcv, r, x, w, gy)."""
    import torch
    s, rcv, r = wl.make_graph(W)
    gen = torch.Generator(device=dev).manual_seed(wl.SEED_X + 100 + seed_offset)
    E = len(s)
    x = torch.randn((W.N, D_in, W.C), generator=gen, device=dev)
    w = torch.randn((E, P, W.C), generator=gen, device=dev).mul_(1.0 / np.sqrt(P))
    gy = torch.randn((W.N, D_out, W.C), generator=gen, device=dev)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return to(s), to(rcv), to(r), x, w, gy


def conv_leg(name, dev, stream, reps, reduce, atomic=True, warmup=3):
    """One of the stated convolution workloads timed kernel by kernel: the
    forward, the deterministic backward and (atomic=True) the atomic
    backward, each median over `reps` launches (max over ranks), with its
    HBM roofline (each kernel's tensors counted once, against the measured
    copy peak) and its FP32 issue fraction (FMAs counted from the CG tables,
    against the FP32 FMA peak at the maximum SM clock)."""
    import torch

    from equivariant_gnn_message_edge_b200 import binding as B
    from equivariant_gnn_message_edge_b200.conv import EqConv
    W = wl.WORKLOADS[name]
    conv = EqConv(W.irreps_in, W.L_sh, W.irreps_out, W.C, all_parity=W.all_parity, per_path=W.per_path)
    P, D_in, D_out = conv.P, conv.D_in, conv.D_out
    with torch.cuda.stream(stream):
        s, rcv, r, x, w, gy = device_inputs(W, D_in, D_out, P, dev)
        g = conv.graph(s, rcv, W.N, stream=stream)
        y, dx, dw, dr = (torch.empty((W.N, D_out, W.C), device=dev), torch.empty_like(x), torch.empty_like(w),
                         torch.empty_like(r))
        nws = B.eqconv_backward_workspace_bytes(conv.plan, g.E)
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
    h = stream.cuda_stream
    modes = [("fwd", None), ("bwd_det", B.EQCONV_DETERMINISTIC)] + ([("bwd_atomic", 0)] if atomic else [])
    times = {}
    for key, flag in modes:
        evs = []
        for k in range(warmup + reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if flag is None:
                B.eqconv_forward(conv.plan, g.c, x, r, w, y, 0, h)
            else:
                B.eqconv_backward(conv.plan, g.c, x, r, w, gy, dx, dw, dr, ws, nws, flag, h)
            b.record(stream)
            if k >= warmup:
                evs.append((a, b))
        stream.synchronize()
        times[key] = reduce(statistics.median([a.elapsed_time(b) for a, b in evs]))
    assert B.eqconv_get_device_error(conv.plan, h) == B.EQCONV_OK
    bc = byte_counts(W.N, g.E, W.C, D_in, D_out, P)
    fma_f, fma_b = fma_counts(conv.paths, B.eqconv_cg_table)
    peak, peak_kind = measured_peak()
    fpk = fp32_peak_tflops()
    out = {"N": W.N, "E": g.E, "C": W.C, "P": P, "irreps": f"{W.irreps_in} -> {W.irreps_out}", "L_sh": W.L_sh,
           "ms": {k: round(v, 4) for k, v in times.items()},
           "fma_per_edge_channel": {"fwd": fma_f, "bwd": fma_b}}
    for key in times:
        nbytes = bc["fwd"] if key == "fwd" else bc["bwd"]
        fma = fma_f if key == "fwd" else fma_b
        sec = times[key] * 1e-3
        gbs = nbytes / sec / 1e9
        tfl = 2.0 * fma * g.E * W.C / sec / 1e12
        out[key] = {"gbps": round(gbs, 1), "edges_per_s": round(g.E / sec, 1),
                    "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                                 "frac": round(gbs / peak, 4), "traffic": None, "algorithmic_bytes": nbytes,
                                 "peak_kind": peak_kind},
                    "roofline_fp32": {"bound": "alu", "achieved": round(tfl, 2), "peak": round(fpk, 2),
                                      "unit": "TFLOP/s", "frac": round(tfl / fpk, 4),
                                      "flop": "2 x FMA per (edge, channel) from the CG tables x E x C"}}
    fb = (bc["fwd"] + bc["bwd"]) / ((times["fwd"] + times["bwd_det"]) * 1e-3) / 1e9
    out["fwd_bwd_gbps_per_kernel_bytes"] = round(fb, 1)
    # every tensor of forward + backward counted once (the edge layout included)
    out["fwd_bwd_gbps_unique_bytes"] = round(bc["step"] / ((times["fwd"] + times["bwd_det"]) * 1e-3) / 1e9, 1)
    out["fwd_bwd_frac_unique"] = round(out["fwd_bwd_gbps_unique_bytes"] / peak, 4)
    del x, w, gy, y, dx, dw, dr, ws, g
    torch.cuda.empty_cache()
    return out


def radial_weights_torch(r, rc, params, P, C):
    """w[E, P, C] = u(d) * MLP(b(d)) with d = |r| in fp32 torch ops (cuBLAS
    GEMMs for the layers): the unfused radial path the water-box step uses
    as its baseline.  The same Bessel basis, C2 polynomial envelope (p = 6)
    and bias-free SiLU MLP as the seeded workload."""
    import torch
    d = torch.linalg.vector_norm(r, dim=1)
    n = torch.arange(1, params[0].shape[0] + 1, device=r.device, dtype=r.dtype)
    x = (d / rc).clamp(0.0, 1.0)
    p = 6.0
    env = (1.0 - (p + 1) * (p + 2) / 2 * x ** 6 + p * (p + 2) * x ** 7 - p * (p + 1) / 2 * x ** 8)
    bes = (2.0 / rc) ** 0.5 * torch.sin(n[None, :] * (np.pi / rc) * d[:, None]) / d.clamp_min(1e-9)[:, None]
    h = torch.nn.functional.silu(bes @ params[0])
    h = torch.nn.functional.silu(h @ params[1])
    return (env[:, None] * (h @ params[2])).view(-1, P, C)


def waterbox_leg(dev, stream, reps, reduce, warmup=3):
    """The MACE(a)-shaped water box step as stated: two stacked conv layers
    (C = 128, L = 3) with radial-MLP weights (8 Bessel functions, 8 -> 64 ->
    64 -> P*C SiLU MLP, a seeded set per layer), layer 2 fed y1 / <degree>,
    an energy-like readout E = <gy, y2>, then the gradient of E with respect
    to the 1503 positions (forces) through both routes of every edge vector
    (the harmonics and the radial weights) and to both MLPs' weights.
    Timed on the device per step, L2 flushed between steps (the box's inputs
    fit in L2)."""
    import torch

    from equivariant_gnn_message_edge_b200 import binding as B
    from equivariant_gnn_message_edge_b200.conv import EqConv, RadialEqConv
    cfg = wl.WATER_BOX
    ins = wl.natural_irreps(cfg["L"])
    C, N, rc = cfg["C"], cfg["n_atoms"], cfg["cutoff"]
    conv = EqConv(ins, cfg["L"], ins, C)
    P = conv.P
    pos, s, rcv, shift, dummy = wl.water_box_system()
    avg = float((~dummy).sum()) / N
    torch.backends.cuda.matmul.allow_tf32 = False
    to = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    with torch.cuda.stream(stream):
        s_d, r_d = to(s, torch.int32), to(rcv, torch.int32)
        g = conv.graph(s_d, r_d, N, stream=stream)
        pos_d, shift_d = to(pos), to(shift)
        s_l, r_l = s_d.long(), r_d.long()
        params = [[to(p) for p in wl.radial_mlp_params(P, C, cfg["hidden"], cfg["n_bessel"], seed=wl.SEED_W + 10 * k)]
                  for k in range(2)]
        x1 = to(wl.features(N, conv.D_in, C, wl.SEED_X))
        readout = to(wl.features(N, conv.D_out, C, wl.SEED_GY))
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    rconv = RadialEqConv(ins, cfg["L"], ins, C, n_basis=cfg["n_bessel"], r_cut=rc)

    def step_unfused():
        p = pos_d.detach().requires_grad_(True)
        Ws = [[t.detach().requires_grad_(True) for t in ps] for ps in params]
        r = p[s_l] - p[r_l] + shift_d
        y1 = conv(g, x1, r, radial_weights_torch(r, rc, Ws[0], P, C))
        y2 = conv(g, y1 / avg, r, radial_weights_torch(r, rc, Ws[1], P, C))
        e = (y2 * readout).sum()
        return torch.autograd.grad(e, [p] + Ws[0] + Ws[1])

    def step_fused():
        p = pos_d.detach().requires_grad_(True)
        Ws = [[t.detach().requires_grad_(True) for t in ps] for ps in params]
        r = p[s_l] - p[r_l] + shift_d
        y1 = rconv(g, x1, r, *Ws[0])
        y2 = rconv(g, y1 / avg, r, *Ws[1])
        e = (y2 * readout).sum()
        return torch.autograd.grad(e, [p] + Ws[0] + Ws[1])

    def timed(fn):
        ms = []
        launches0 = B.eqconv_launch_count()
        with torch.cuda.stream(stream):
            for k in range(warmup + reps):
                flush.fill_(k & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                if k >= warmup:
                    ms.append((a, b))
        stream.synchronize()
        assert B.eqconv_get_device_error(conv.plan, stream.cuda_stream) == B.EQCONV_OK
        launches = (B.eqconv_launch_count() - launches0) // (warmup + reps)
        return reduce(statistics.median([a.elapsed_time(b) for a, b in ms])), launches

    t_u, _ = timed(step_unfused)
    t_f, l_f = timed(step_fused)
    return {"atoms": N, "edges": int(len(s)), "dummy_edges": int(dummy.sum()), "C": C, "L": cfg["L"], "P": P,
            "ms_per_step": round(t_f, 4), "unfused_ms_per_step": round(t_u, 4),
            "speedup_vs_unfused": round(t_u / t_f, 2), "libeqconv_launches_per_step": int(l_f),
            "fused": "libeqconv eqconv_forward_radial / eqconv_backward_radial per layer (radial MLP on the "
                     "chip: w and dw never in memory) + torch autograd for positions -> edge vectors and the "
                     "readout",
            "unfused": "radial MLP in fp32 torch ops (cuBLAS GEMMs, TF32 off) writing w [E][P][C] to HBM per "
                       "layer + libeqconv forward/backward (deterministic) + torch autograd glue",
            "step": "2 conv layers forward + gradient of <gy, y2> w.r.t. positions (forces) and MLP weights; "
                    "L2 flushed between steps"}


def radial_leg(name, dev, stream, reps, reduce, warmup=3):
    """The convolution of workload `name` with radial-MLP weights (8 Bessel
    functions, 8 -> 64 -> 64 -> P*C SiLU MLP, 5 A cutoff): the fused path
    (eqconv_forward_radial / eqconv_backward_radial: w and dw never in
    memory) against the unfused one (the same MLP in fp32 torch ops writing
    w to memory, libeqconv's forward and backward, torch autograd for the
    MLP), each forward and forward+backward."""
    import torch

    from equivariant_gnn_message_edge_b200 import binding as B
    from equivariant_gnn_message_edge_b200.conv import EqConv, RadialEqConv
    W = wl.WORKLOADS[name]
    rc, nb = 5.0, 8
    rconv = RadialEqConv(W.irreps_in, W.L_sh, W.irreps_out, W.C, n_basis=nb, r_cut=rc)
    conv = EqConv(W.irreps_in, W.L_sh, W.irreps_out, W.C)
    P, D_in, D_out, C = conv.P, conv.D_in, conv.D_out, W.C
    torch.backends.cuda.matmul.allow_tf32 = False
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    with torch.cuda.stream(stream):
        s, rcv, r = wl.make_graph(W)
        E = len(s)
        s_d, r_d, rv = to(s), to(rcv), to(r)
        g = conv.graph(s_d, r_d, W.N, stream=stream)
        gen = torch.Generator(device=dev).manual_seed(wl.SEED_X + 200)
        x = torch.randn((W.N, D_in, C), generator=gen, device=dev)
        gy = torch.randn((W.N, D_out, C), generator=gen, device=dev)
        params = [to(p) for p in wl.radial_mlp_params(P, C, 64, nb)]
        y = torch.empty((W.N, D_out, C), device=dev)
        fws_n = B.eqconv_forward_radial_workspace_bytes(rconv.plan, W.N, E)
        bws_n = B.eqconv_backward_radial_workspace_bytes(rconv.plan, W.N, E)
        fws = torch.empty(fws_n, dtype=torch.uint8, device=dev)
        bws = torch.empty(bws_n, dtype=torch.uint8, device=dev)
        dx, dr = torch.empty_like(x), torch.empty_like(rv)
        gW = [torch.empty_like(p) for p in params]
    h = stream.cuda_stream

    def fused_fwd():
        B.eqconv_forward_radial(rconv.plan, g.c, x, rv, *params, nb, rc, y, fws, fws_n, h)

    def fused_bwd():
        B.eqconv_backward_radial(rconv.plan, g.c, x, rv, *params, nb, rc, gy, dx, dr, *gW, bws, bws_n, h)

    def unfused_fwd():
        w = radial_weights_torch(rv, rc, params, P, C)
        B.eqconv_forward(conv.plan, g.c, x, rv, w, y, 0, h)

    def unfused_fwd_bwd():
        xr = x.detach().requires_grad_(True)
        rr = rv.detach().requires_grad_(True)
        Ws = [p.detach().requires_grad_(True) for p in params]
        yy = conv(g, xr, rr, radial_weights_torch(rr, rc, Ws, P, C))
        return torch.autograd.grad(yy, [xr, rr] + Ws, gy)

    def timed(fn):
        out = []
        with torch.cuda.stream(stream):
            for k in range(warmup + reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                if k >= warmup:
                    out.append((a, b))
        stream.synchronize()
        return reduce(statistics.median([a.elapsed_time(b) for a, b in out]))

    t_ff, t_fb = timed(fused_fwd), timed(fused_bwd)
    t_uf, t_ufb = timed(unfused_fwd), timed(unfused_fwd_bwd)
    assert B.eqconv_get_device_error(rconv.plan, h) == B.EQCONV_OK
    flop = 6.0 * E * 64 * P * C          # 3 fp16 products, 2 flop per multiply-add, per forward GEMM
    peak_tc = measured_tensor_peak()
    out = {"N": W.N, "E": E, "C": C, "P": P, "radial": "8 Bessel, 8 -> 64 -> 64 -> P*C SiLU MLP, 5 A cutoff",
           "fused_ms": {"fwd": round(t_ff, 4), "bwd": round(t_fb, 4), "fwd_bwd": round(t_ff + t_fb, 4)},
           "unfused_ms": {"fwd": round(t_uf, 4), "fwd_bwd": round(t_ufb, 4)},
           "speedup_fwd": round(t_uf / t_ff, 2), "speedup_fwd_bwd": round(t_ufb / (t_ff + t_fb), 2),
           "roofline_fwd_tensor": {"bound": "tensor", "achieved": round(flop / (t_ff * 1e-3) / 1e12, 1),
                                   "peak": peak_tc[0], "unit": "TFLOP/s",
                                   "frac": round(flop / (t_ff * 1e-3) / 1e12 / peak_tc[0], 4),
                                   "flop": "6 E 64 P C: the last layer's three fp16 products (the whole fused "
                                           "forward timed)", "peak_kind": peak_tc[1]},
           "unfused": "radial MLP in fp32 torch ops (cuBLAS, TF32 off) writing w to memory + libeqconv "
                      "forward/backward + torch autograd for the MLP"}
    del fws, bws, x, gy, y, dx, dr
    torch.cuda.empty_cache()
    return out


def measured_tensor_peak():
    """Dense f16 / bf16 tensor peak (TFLOP/s): the measured cuBLAS bf16 burst
    figure (f16 runs at the bf16 rate), else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (bf16 burst; f16 has the same rate)"
    except Exception:
        return 1590.0, "fallback"


def dbl_bytes(N, E, C, D_in, D_out, P, part_bytes):
    """Algorithmic bytes of one double backward: receiver pass, sender pass
    and r epilogue, each kernel's inputs and outputs counted once."""
    t = tensor_bytes(N, E, C, D_in, D_out, P)
    recv = 2 * t["x"] + 2 * t["r"] + 2 * t["w"] + t["recv_ptr"] + t["recv_perm"] + t["senders"] + t["y"]
    send = (2 * t["x"] + 2 * t["r"] + 2 * t["w"] + t["gy"] + t["send_ptr"] + t["send_perm"] + t["receivers"] +
            t["dx"] + t["dw"] + part_bytes)
    epi = part_bytes + 3 * t["r"]
    return recv + send + epi


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# --------------------------------------------------------------------- inputs

class Inputs:
    """Seeded synthetic workload on the host (pinned when asked)."""

    def __init__(self, name, P, D_in, D_out, pinned):
        import torch
        W = wl.WORKLOADS[name]
        self.W = W
        s, rcv, r = wl.make_graph(W)
        self.N, self.E, self.C = W.N, len(s), W.C
        mk = (lambda shape, dt: torch.empty(shape, dtype=dt, pin_memory=True)) if pinned else \
            (lambda shape, dt: torch.empty(shape, dtype=dt))
        self.senders = mk((self.E,), torch.int32)
        self.receivers = mk((self.E,), torch.int32)
        self.r = mk((self.E, 3), torch.float32)
        self.senders.numpy()[:] = s
        self.receivers.numpy()[:] = rcv
        self.r.numpy()[:] = r
        self.x = mk((W.N, D_in, W.C), torch.float32)
        self.x.numpy()[:] = wl.features(W.N, D_in, W.C, wl.SEED_X)
        self.gy = mk((W.N, D_out, W.C), torch.float32)
        self.gy.numpy()[:] = wl.features(W.N, D_out, W.C, wl.SEED_GY)
        self.w = mk((self.E, P, W.C), torch.float32)
        if W.kind == "waterbox":           # radial-MLP weights, zero on the padding edges
            self.w.numpy()[:] = wl.water_box_weights(P, W.C)
        else:
            wl.weights_into(self.w.numpy())


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.monotonic(), ln.strip()))

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self, window=None):
        """Median SM clock and the throttle reasons seen; restricted to the
        timed window when it holds at least 2 samples (else warm-up + timed)."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        scope = "warmup+timed"
        if window is not None:
            inside = [(t, ln) for t, ln in lines if window[0] <= t <= window[1]]
            if len(inside) >= 2:
                lines, scope = inside, "timed"
        for _, ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "scope": scope}


# --------------------------------------------------------------------- ranks

def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(bytes_per_step: int, steps: int, world: int, t_max_ms: float) -> float:
    """Whole-job throughput: every rank's bytes over the slowest rank's time."""
    return bytes_per_step * steps * world / (t_max_ms * 1e-3) / 1e9


# --------------------------------------------------------------------- native

def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from equivariant_gnn_message_edge_b200 import binding as B
    from equivariant_gnn_message_edge_b200.conv import EqConv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    W = wl.WORKLOADS[args.workload]
    conv = EqConv(W.irreps_in, W.L_sh, W.irreps_out, W.C, all_parity=W.all_parity, per_path=W.per_path)
    if args.vec:
        conv.set_vec(*[int(v) for v in args.vec.split(",")])
    if args.gather_budget_mib is not None:
        conv.set_gather_budget(int(args.gather_budget_mib * (1 << 20)))
    P, D_in, D_out = conv.P, conv.D_in, conv.D_out
    inp = Inputs(args.workload, P, D_in, D_out, pinned=True)
    N, E, C = inp.N, inp.E, inp.C
    bc = byte_counts(N, E, C, D_in, D_out, P)

    stream = torch.cuda.Stream(device=dev)

    class DeviceSet:
        """Device copies of one step's inputs, its edge layout and outputs."""

        def __init__(self):
            with torch.cuda.stream(stream):
                self.s = inp.senders.to(dev, non_blocking=True)
                self.r = inp.receivers.to(dev, non_blocking=True)
                self.x = inp.x.to(dev, non_blocking=True)
                self.rv = inp.r.to(dev, non_blocking=True)
                self.w = inp.w.to(dev, non_blocking=True)
                self.gy = inp.gy.to(dev, non_blocking=True)
                self.g = conv.graph(self.s, self.r, N, stream=stream)
                self.y = torch.empty((N, D_out, C), dtype=torch.float32, device=dev)
                self.dx = torch.empty_like(self.x)
                self.dw = torch.empty_like(self.w)
                self.dr = torch.empty_like(self.rv)
            stream.synchronize()

    ds0 = DeviceSet()
    gws_n = B.eqconv_graph_workspace_bytes(N, E)
    gws = torch.empty(max(gws_n, 1), dtype=torch.uint8, device=dev)
    bws_n = B.eqconv_backward_workspace_bytes(conv.plan, E)
    bws = torch.empty(max(bws_n, 1), dtype=torch.uint8, device=dev)
    sh = stream.cuda_stream

    def step(ev=None, ds=ds0, st=stream):
        h = st.cuda_stream
        if ev is not None:
            ev[0].record(st)
        B.eqconv_graph_build(conv.plan, ds.g.c, gws, gws_n, h)
        if ev is not None:
            ev[1].record(st)
        B.eqconv_forward(conv.plan, ds.g.c, ds.x, ds.rv, ds.w, ds.y, 0, h)
        if ev is not None:
            ev[2].record(st)
        B.eqconv_backward(conv.plan, ds.g.c, ds.x, ds.rv, ds.w, ds.gy, ds.dx, ds.dw, ds.dr, bws, bws_n,
                          B.EQCONV_DETERMINISTIC, h)
        if ev is not None:
            ev[3].record(st)

    def barrier():
        if world > 1:
            dist.barrier()

    gpu_id = None
    try:
        gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_id.startswith("GPU-"):
            gpu_id = "GPU-" + gpu_id
    except Exception:
        gpu_id = None
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id) as clk:
        time.sleep(0.3)                      # let the sampler start
        for _ in range(args.warmup):
            step()
        stream.synchronize()
        assert B.eqconv_get_device_error(conv.plan, sh) == B.EQCONV_OK
        barrier()
        torch.cuda.synchronize(dev)
        launches0 = B.eqconv_launch_count()
        w0 = time.monotonic()
        t0.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        w1 = time.monotonic()
        launches = B.eqconv_launch_count() - launches0
        barrier()
    total_ms = t0.elapsed_time(t1)
    graph_ms = [e[0].elapsed_time(e[1]) for e in evs]
    fwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    bwd_ms = [e[2].elapsed_time(e[3]) for e in evs]
    t_max = reduce_max(total_ms, world, dev)

    # non-deterministic backward, timed separately (not part of the step)
    nd_ms = []
    for _ in range(max(2, args.steps // 2)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        B.eqconv_backward(conv.plan, ds0.g.c, ds0.x, ds0.rv, ds0.w, ds0.gy, ds0.dx, ds0.dw, ds0.dr, bws, bws_n,
                          0, sh)
        b.record(stream)
        nd_ms.append((a, b))
    stream.synchronize()
    nd_ms = [a.elapsed_time(b) for a, b in nd_ms[1:]]

    # double backward (VJP of the backward), timed separately (not part of the step)
    dbl = None
    dws_n = B.eqconv_double_backward_workspace_bytes(conv.plan, E)
    if W.all_parity is False and W.per_path is False and not args.no_double_backward:
        gen = torch.Generator(device=dev).manual_seed(wl.SEED_GY + 1)
        with torch.cuda.stream(stream):
            cot_a = torch.randn(ds0.x.shape, generator=gen, device=dev)
            cot_b = torch.randn(ds0.w.shape, generator=gen, device=dev)
            cot_q = torch.randn(ds0.rv.shape, generator=gen, device=dev)
            outs = (torch.empty_like(ds0.x), torch.empty_like(ds0.w), torch.empty_like(ds0.gy),
                    torch.empty_like(ds0.rv))
            dws = torch.empty(max(dws_n, 1), dtype=torch.uint8, device=dev)
        dbl_ev = []
        for k in range(max(3, args.steps // 2) + 1):
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            B.eqconv_double_backward(conv.plan, ds0.g.c, ds0.x, ds0.rv, ds0.w, ds0.gy, cot_a, cot_b, cot_q,
                                     *outs, dws, dws_n, sh)
            a1.record(stream)
            dbl_ev.append((a0, a1))
        stream.synchronize()
        assert B.eqconv_get_device_error(conv.plan, sh) == B.EQCONV_OK
        dbl_ms = [a.elapsed_time(b) for a, b in dbl_ev[1:]]
        nbytes = dbl_bytes(N, E, C, D_in, D_out, P, dws_n)
        dbl_med = reduce_max(statistics.median(dbl_ms), world, dev)     # max over ranks
        dbl = {"ms": round(dbl_med, 4), "gbps": round(nbytes / (dbl_med * 1e-3) / 1e9, 1),
               "frac_of_measured_hbm": round(nbytes / (dbl_med * 1e-3) / 1e9 / measured_peak()[0], 4),
               "algorithmic_bytes": nbytes, "launches_per_call": 3,
               "bytes": "per kernel: receiver pass, sender pass, r epilogue, each tensor once per kernel"}
        del cot_a, cot_b, cot_q, outs, dws

    # node-local channel-diagonal product on 4N nodes of the same irreps (inputs
    # well above L2), forward and backward, timed separately
    nprod = None
    if not W.all_parity and not args.no_node_product:
        nprod = time_node_product(W, 4 * N, dev, stream, max(3, args.steps // 2),
                                  lambda t: reduce_max(t, world, dev))
    # symmetric contraction of correlation order 2 (4 species) on 4N nodes
    symc = None
    if not W.all_parity and not W.per_path and not args.no_node_product:
        symc = time_symmetric_contraction(W, 4 * N, dev, stream, max(3, args.steps // 2),
                                          lambda t: reduce_max(t, world, dev))

    # End to end through the public API with host buffers (pinned), copies
    # timed: every step uploads its inputs and downloads its results.  Steps
    # are pipelined over two device sets and three streams, so step k's
    # upload, step k-1's compute and step k-2's download overlap.
    e2e = None
    if not args.no_e2e:
        sets = [ds0, DeviceSet()]
        outs_h = [(torch.empty((N, D_out, C), dtype=torch.float32, pin_memory=True),
                   torch.empty((N, D_in, C), dtype=torch.float32, pin_memory=True),
                   torch.empty((E, P, C), dtype=torch.float32, pin_memory=True),
                   torch.empty((E, 3), dtype=torch.float32, pin_memory=True)) for _ in range(2)]
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        free = [None, None]     # event: the set's previous download has finished

        def e2e_step(k):
            ds, oh = sets[k % 2], outs_h[k % 2]
            if free[k % 2] is not None:
                up.wait_event(free[k % 2])
            with torch.cuda.stream(up):
                for dst, src in ((ds.s, inp.senders), (ds.r, inp.receivers), (ds.x, inp.x), (ds.rv, inp.r),
                                 (ds.w, inp.w), (ds.gy, inp.gy)):
                    dst.copy_(src, non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(up)
            stream.wait_event(loaded)
            step(ds=ds, st=stream)
            done = torch.cuda.Event()
            done.record(stream)
            down.wait_event(done)
            with torch.cuda.stream(down):
                for dst, src in zip(oh, (ds.y, ds.dx, ds.dw, ds.dr)):
                    dst.copy_(src, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(down)
            free[k % 2] = ev

        e2e_steps = max(3, min(args.steps, 6))
        for k in range(2):
            e2e_step(k)
        torch.cuda.synchronize(dev)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(up)
        for k in range(e2e_steps):
            e2e_step(k)
        down.wait_event(free[(e2e_steps - 1) % 2])
        b.record(down)
        torch.cuda.synchronize(dev)
        e_ms = reduce_max(a.elapsed_time(b), world, dev)
        e2e = {"value": round(aggregate_gbs(bc["step"], e2e_steps, world, e_ms), 2), "unit": UNIT,
               "h2d_bytes_per_step": bc["h2d"], "d2h_bytes_per_step": bc["d2h"],
               "ms_per_step": round(e_ms / e2e_steps, 3),
               "pipeline": "2 device sets; upload / compute / download streams overlap across steps"}
        del sets[1]

    # the other stated workloads, timed kernel by kernel after the main
    # step: lmax=3 with both backward modes, the channel sweep at lmax=2, and
    # the water-box step
    legs = {}
    want = set(args.legs.split(",")) if args.legs else set()
    red = lambda t: reduce_max(t, world, dev)
    reps = max(5, args.steps // 2)
    if "lmax3" in want:
        legs["lmax3"] = conv_leg("lmax3", dev, stream, reps, red, atomic=True)
    if "sweep" in want:
        legs["sweepC"] = [conv_leg(f"sweepC{c}", dev, stream, reps, red, atomic=False)
                          for c in (64, 128, 256, 512, 1024)]
    if "waterbox" in want:
        legs["waterbox"] = waterbox_leg(dev, stream, reps, red)
    if "radial" in want:   # on the run's own graph when it is an lmax=2 one (smaller profiling runs)
        legs["radial_lmax2"] = radial_leg(args.workload if args.workload.startswith("lmax2") else "lmax2", dev,
                                          stream, reps, red)

    peak, peak_kind = measured_peak()
    ms_step = t_max / args.steps
    med = statistics.median
    value = aggregate_gbs(bc["step"], args.steps, world, t_max)           # unique bytes of the step
    kernel_gbs = aggregate_gbs(bc["kernels"], args.steps, world, t_max)   # each kernel's own tensors
    fwd_gbs = bc["fwd"] / (med(fwd_ms) * 1e-3) / 1e9
    bwd_gbs = bc["bwd"] / (med(bwd_ms) * 1e-3) / 1e9
    fb_gbs = (bc["fwd"] + bc["bwd"]) / ((med(fwd_ms) + med(bwd_ms)) * 1e-3) / 1e9
    fwdbwd_unique_gbs = bc["step"] / ((med(fwd_ms) + med(bwd_ms)) * 1e-3) / 1e9
    bwd_avg = sum(bwd_ms) / len(bwd_ms)
    fwd_avg = sum(fwd_ms) / len(fwd_ms)
    layout = f" (per-path blocks, D_out={D_out})" if W.per_path else ""
    # ncu counters hold for the default launch configuration only
    traffic = load_traffic(W.name) if not (args.vec or args.gather_budget_mib is not None) else {}
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded NumPy PCG64)",
        "config": step_config(W, N, E, C, D_in, D_out, P, world, layout),
        "kernel_bytes_step_gbps": round(kernel_gbs, 1),
        "kernel_bytes_per_step": bc["kernels"],
        "fwd_gbps": round(fwd_gbs, 1), "bwd_gbps": round(bwd_gbs, 1),
        "fwd_bwd_gbps_unique": round(fwdbwd_unique_gbs, 1),
        "hbm_frac_fwd_bwd_unique": round(fwdbwd_unique_gbs / peak, 4),
        "fwd_bwd_gbps_per_kernel_bytes": round(fb_gbs, 1),
        "hbm_frac_fwd_bwd_per_kernel_bytes": round(fb_gbs / peak, 4),
        "edges_per_s_fwd": round(E / (med(fwd_ms) * 1e-3), 1),
        "edges_per_s_fwd_bwd": round(E / ((med(fwd_ms) + med(bwd_ms)) * 1e-3), 1),
        "ms": {"graph": round(med(graph_ms), 4), "fwd": round(med(fwd_ms), 4), "bwd_det": round(med(bwd_ms), 4),
               "bwd_atomic": round(med(nd_ms), 4) if nd_ms else None},
        "roofline": {"bound": "hbm",
                     "kernel": "eqconv_bwd_kernel (deterministic; dr finished in-kernel when one channel "
                               "tile covers C, else by eqconv_dr_epilogue)",
                     "achieved": round(bc["bwd"] / (bwd_avg * 1e-3) / 1e9, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(bc["bwd"] / (bwd_avg * 1e-3) / 1e9 / peak, 4),
                     "traffic": traffic.get("bwd"), "algorithmic_bytes": bc["bwd"], "peak_kind": peak_kind},
        "roofline_fwd": {"bound": "hbm", "kernel": "eqconv_fwd_kernel",
                         "achieved": round(bc["fwd"] / (fwd_avg * 1e-3) / 1e9, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(bc["fwd"] / (fwd_avg * 1e-3) / 1e9 / peak, 4), "traffic": traffic.get("fwd"),
                         "algorithmic_bytes": bc["fwd"]},
        "double_backward": dbl,
        "node_product": nprod,
        "symmetric_contraction": symc,
        "workloads": legs,
        "gpu_launches": int(launches),
        "clocks": clk.summary((w0, w1)),
    }
    if e2e:
        result["e2e"] = e2e
    return result, inp, (N, E, C, D_in, D_out, P)


def step_config(W, N, E, C, D_in, D_out, P, world, layout=""):
    """The `config` object of the JSON line; the same for both arms."""
    bc_step = byte_counts(N, E, C, D_in, D_out, P)["step"]
    return {
        "workload": f"{W.name}: N={N}, C={C}, E={E}, irreps {W.irreps_in} -> {W.irreps_out}{layout}, L_sh={W.L_sh}, "
                    f"P={P}, " + (f"water box: {W.N} atoms, {W.box:g} A periodic cube, cutoff {W.cutoff:g} A, "
                                  f"10% zero-weight padding edges, radial-MLP weights (one conv layer)"
                                  if W.kind == "waterbox" else
                                  f"in-degree Poisson({W.mean_degree:g}), uniform senders"),
        "step": "graph build (recv+send CSR) + fused forward + fused deterministic backward",
        "l2": "inputs larger than L2 (w alone is %.1f GB)" % (4 * E * P * C / 1e9),
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        "bytes_per_step": bc_step,
        "bytes": "unique: every tensor the step reads or writes (senders, receivers, CSR arrays, x, r, w, gy, "
                 "y, dx, dw, dr) counted once over the whole step; GB/s = bytes / device time",
    }


def kernel_code_hash(paths):
    """sha256 of the kernel sources with comments and blank lines removed, so
    that a comment edit does not mark the ncu counters stale but any code
    change does."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
        h.update("\n".join(lines).encode())
    return h.hexdigest()


def load_traffic(workload):
    """DRAM bytes per launch of the forward and the deterministic backward
    for `workload` from the committed ncu summary; empty (so the roofline's
    traffic is null) when absent, when that workload was not captured, or
    when the kernel code has changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if kernel_code_hash(d["kernel_sources"]) != d["kernel_code_sha256"]:
            return {}
        return d["workloads"].get(workload, {})
    except Exception:
        return {}


# --------------------------------------------------------------------- oracle

def oracle_sample_step(name, n_recv, D_in, D_out, P, x=None, gy=None, nthreads=0):
    """The whole path on the CPU oracle for the in-edges of receivers
    0..n_recv-1 of the workload: CSR of the sample, harmonics, forward rows,
    backward dx rows, dw/gY per edge, dr.  Returns (seconds, sample edges)."""
    from oracle import conv as oconv
    from oracle.csr import csr
    from oracle.sh import sh
    W = wl.WORKLOADS[name]
    s, rcv, r = wl.make_graph(W)
    k = int(np.searchsorted(rcv, n_recv))      # receiver-sorted workload
    s_s, r_s, rv_s = s[:k], rcv[:k], r[:k]
    w_s = wl.weights(k, P, W.C)
    if x is None:
        x = wl.features(W.N, D_in, W.C, wl.SEED_X)
    if gy is None:
        gy = wl.features(W.N, D_out, W.C, wl.SEED_GY)
    prob = oconv.Problem(W.irreps_in, W.L_sh, W.irreps_out, W.C, per_path=W.per_path)
    t = time.perf_counter()
    rp, rperm = csr(r_s, W.N)
    sp, sperm = csr(s_s, W.N)
    Y = sh(rv_s, W.L_sh)
    oconv.forward(prob, rp, rperm, s_s, Y, x, w_s, rows=np.unique(r_s), nthreads=nthreads)
    oconv.backward_dx(prob, sp, sperm, r_s, Y, gy, w_s, rows=np.unique(s_s), nthreads=nthreads)
    _, gY = oconv.backward_edges(prob, s_s, r_s, Y, x, gy, w_s, nthreads=nthreads)
    oconv.dr_from_gY(rv_s, gY, W.L_sh)
    return time.perf_counter() - t, k


def cpu_baseline(name, D_in, D_out, P, target_s, bytes_step, E_full):
    from oracle import conv as oconv
    W = wl.WORKLOADS[name]
    x = wl.features(W.N, D_in, W.C, wl.SEED_X)
    gy = wl.features(W.N, D_out, W.C, wl.SEED_GY)
    n_recv, t = 16, 0.0
    while n_recv < W.N:                       # grow the sample until it is long enough to scale
        t, k = oracle_sample_step(name, n_recv, D_in, D_out, P, x, gy)
        if t >= target_s / 8:
            break
        n_recv = min(W.N, n_recv * 4)
    n_recv = int(min(W.N, max(16, n_recv * target_s / max(t, 1e-3))))
    t, k = oracle_sample_step(name, n_recv, D_in, D_out, P, x, gy)
    frac = k / E_full
    return {"value": round(bytes_step * frac / t / 1e9, 4), "unit": UNIT, "cores": oconv.max_threads(),
            "kind": "oracle", "edges_per_s": round(k / t, 1), "seconds": round(t, 2),
            "sample": f"in-edges of receivers 0..{n_recv - 1} ({k} of {E_full} edges): CSR, SH, forward rows, "
                      f"backward dx/dw/dr; bytes scaled by the edge fraction {frac:.5f}"}


def run_reference(args, rank, world):
    """CPU oracle as the reference arm: each step is a bounded sample."""
    from oracle import build as obuild
    from oracle import conv as oconv
    obuild.build()
    W = wl.WORKLOADS[args.workload]
    prob = oconv.Problem(W.irreps_in, W.L_sh, W.irreps_out, W.C, per_path=W.per_path)
    s, rcv, r = wl.make_graph(W)
    E = len(s)
    bc = byte_counts(W.N, E, W.C, prob.D_in, prob.D_out, prob.P)
    x = wl.features(W.N, prob.D_in, W.C, wl.SEED_X)
    gy = wl.features(W.N, prob.D_out, W.C, wl.SEED_GY)
    t0, _ = oracle_sample_step(args.workload, 16, prob.D_in, prob.D_out, prob.P, x, gy)
    budget = max(1.0, args.ref_seconds / max(1, args.steps + args.warmup))
    n_recv = int(min(W.N, max(16, 16 * budget / max(t0, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample_step(args.workload, n_recv, prob.D_in, prob.D_out, prob.P, x, gy)
    tot, k = 0.0, 0
    for _ in range(args.steps):
        t, k = oracle_sample_step(args.workload, n_recv, prob.D_in, prob.D_out, prob.P, x, gy)
        tot += t
    frac = k / E
    value = bc["step"] * frac * args.steps / tot / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot / args.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded NumPy PCG64)",
        "config": step_config(W, W.N, E, W.C, prob.D_in, prob.D_out, prob.P, world,
                              f" (per-path blocks, D_out={prob.D_out})" if W.per_path else ""),
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oconv.max_threads(), "kind": "oracle",
                         "sample": f"in-edges of receivers 0..{n_recv - 1} ({k} of {E} edges) per step; "
                                   f"bytes scaled by {frac:.5f}"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


# --------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="lmax2", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--vec", default=None, help="fwd,bwd channel vector widths (2 or 4)")
    ap.add_argument("--gather-budget-mib", type=float, default=None,
                    help="L2 budget of one gather band in MiB (0: no banding)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-double-backward", action="store_true")
    ap.add_argument("--no-node-product", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    ap.add_argument("--legs", default="lmax3,sweep,waterbox,radial",
                    help="other stated workloads to time after the main step (comma list of lmax3, sweep, "
                         "waterbox, radial; empty for none)")
    ap.add_argument("--nodes", type=int, default=None,
                    help="override the workload's node count (smaller profiling captures)")
    args = ap.parse_args()
    if args.nodes:
        import dataclasses
        base = wl.WORKLOADS[args.workload]
        name = f"{base.name}_N{args.nodes}"
        wl.WORKLOADS[name] = dataclasses.replace(base, name=name, N=args.nodes)
        args.workload = name
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    try:
        result, inp, dims = run_native(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            from oracle import build as obuild
            obuild.build()
            N, E, C, D_in, D_out, P = dims
            result["cpu_baseline"] = cpu_baseline(args.workload, D_in, D_out, P, args.cpu_seconds,
                                                  byte_counts(N, E, C, D_in, D_out, P)["step"], E)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
