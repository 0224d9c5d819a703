"""Seeded synthetic inputs for the equivariant convolution.

This module draws graphs, edge vectors, features, weights and output
gradients.  It holds none of the convolution's arithmetic, so both the CUDA
library's tests/benchmarks and the CPU oracle can be fed from it.

Workloads (shapes from the e3j page, Table 1 and Table 2):

* ``tiny``   - 256 atoms uniform in a 10 A periodic cube, cutoff 3.5 A, both
               edge directions, no self edges, receiver-sorted (stable on
               sender); C=32, irreps 0e+1o -> 0e+1o+2e, L_sh=2.
* ``lmax2``  - N=32768, C=128, in-degree Poisson(45), uniform random senders,
               receiver-sorted; random directions, |r| ~ U[0.5, 5] A;
               irreps 0e+1o+2e, L_sh=2 (Table 1 setting, N*C = 2^22).
* ``lmax3``  - N=16384, C=128, same graph law; irreps 0e+1o+2e+3o, L_sh=3
               (Table 1 setting, N*C = 2^21).
* ``sweepC`` - lmax=2 with N = 2^22 / C, C in {64, ..., 1024}.

Distributions: features and output gradients N(0, 1) fp32; weights
N(0, 1/P) fp32 (variance 1/P).  Seeds: graph 1001, edge vectors 1002,
features 1003, weights 1004, output gradients 1005 (NumPy PCG64).  Weights are
drawn row by row in edge order, so the first k edges' weights are a prefix of
the full draw (used to build bounded samples of the full workload).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

SEED_GRAPH, SEED_R, SEED_X, SEED_W, SEED_GY = 1001, 1002, 1003, 1004, 1005


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    C: int
    irreps_in: str
    L_sh: int
    irreps_out: str
    kind: str            # "box" or "poisson"
    mean_degree: float = 45.0
    box: float = 10.0
    cutoff: float = 3.5
    all_parity: bool = False   # outputs of both parities (irreps_out a both-parity prefix)
    per_path: bool = False     # one output block per path (no summation over paths)


def _natural(L: int) -> str:
    return "+".join(f"{l}{'e' if l % 2 == 0 else 'o'}" for l in range(L + 1))


WORKLOADS = {
    "tiny": Workload("tiny", 256, 32, "0e+1o", 2, _natural(2), "box"),
    "lmax2": Workload("lmax2", 32768, 128, _natural(2), 2, _natural(2), "poisson"),
    "lmax3": Workload("lmax3", 16384, 128, _natural(3), 3, _natural(3), "poisson"),
}
# output variants of the lmax=2 / lmax=3 graphs: per-path blocks (MACE's
# "mid" irreps) and both-parity outputs
WORKLOADS["lmax2_perpath"] = Workload("lmax2_perpath", 32768, 128, _natural(2), 2, _natural(2), "poisson",
                                      per_path=True)
WORKLOADS["lmax2_both"] = Workload("lmax2_both", 32768, 128, _natural(2), 2, "0e+1o+1e+2e+2o", "poisson",
                                   all_parity=True)
WORKLOADS["lmax3_perpath"] = Workload("lmax3_perpath", 16384, 128, _natural(3), 3, _natural(3), "poisson",
                                      per_path=True)
for _C in (64, 128, 256, 512, 1024):
    WORKLOADS[f"sweepC{_C}"] = Workload(f"sweepC{_C}", (1 << 22) // _C, _C, _natural(2), 2,
                                        _natural(2), "poisson")


def natural_irreps(L: int) -> str:
    """'0e+1o+...' up to L (natural parity)."""
    return _natural(L)


def both_parity_irreps(L: int) -> str:
    """'0e+1o+1e+2e+2o+...' up to L: for every l >= 1 the natural-parity irrep
    and then the other one (0o is left out: no path from natural-parity inputs
    reaches it)."""
    names = ["0e"]
    for l in range(1, L + 1):
        nat = "e" if l % 2 == 0 else "o"
        names += [f"{l}{nat}", f"{l}{'o' if nat == 'e' else 'e'}"]
    return "+".join(names)


def poisson_graph(N: int, mean_degree: float, seed: int = SEED_GRAPH):
    """Receiver-sorted random graph: deg_i ~ Poisson(mean), senders uniform."""
    rng = np.random.default_rng(seed)
    deg = rng.poisson(mean_degree, size=N)
    receivers = np.repeat(np.arange(N, dtype=np.int32), deg)
    senders = rng.integers(0, N, size=receivers.size, dtype=np.int64).astype(np.int32)
    return senders, receivers


def random_edge_vectors(E: int, seed: int = SEED_R, lo: float = 0.5, hi: float = 5.0):
    rng = np.random.default_rng(seed)
    d = rng.standard_normal((E, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    length = rng.uniform(lo, hi, size=E)
    return (d * length[:, None]).astype(np.float32)


def periodic_box_graph(n_atoms: int, box: float, cutoff: float, seed: int = SEED_GRAPH):
    """All ordered pairs (receiver i, sender j), i != j, within the cutoff under
    the minimum-image convention; edge vector r = pos[j] - pos[i] (minimum
    image).  Sorted by receiver, stable on sender."""
    rng = np.random.default_rng(seed)
    pos = rng.uniform(0.0, box, size=(n_atoms, 3))
    d = pos[None, :, :] - pos[:, None, :]           # [i, j] = pos[j] - pos[i]
    d -= box * np.round(d / box)
    dist = np.linalg.norm(d, axis=-1)
    mask = (dist < cutoff) & ~np.eye(n_atoms, dtype=bool)
    recv, send = np.nonzero(mask)                    # row-major: sorted by i then j
    r = d[recv, send].astype(np.float32)
    return send.astype(np.int32), recv.astype(np.int32), r


def features(rows: int, D: int, C: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.standard_normal((rows, D, C), dtype=np.float32)


def weights(E: int, P: int, C: int, seed: int = SEED_W, chunk_edges: int = 1 << 16) -> np.ndarray:
    """w[E, P, C] ~ N(0, 1/P), drawn in edge order in chunks (prefix-stable)."""
    rng = np.random.default_rng(seed)
    out = np.empty((E, P, C), dtype=np.float32)
    scale = np.float32(1.0 / np.sqrt(P))
    for a in range(0, E, chunk_edges):
        b = min(E, a + chunk_edges)
        blk = out[a:b]
        rng.standard_normal(blk.shape, dtype=np.float32, out=blk)
        blk *= scale
    return out


def weights_into(out: np.ndarray, seed: int = SEED_W, chunk_edges: int = 1 << 16) -> np.ndarray:
    """Fill a preallocated fp32 array [E, P, C] (e.g. pinned host memory) with
    the same values as ``weights(E, P, C, seed)``."""
    E, P, C = out.shape
    rng = np.random.default_rng(seed)
    scale = np.float32(1.0 / np.sqrt(P))
    for a in range(0, E, chunk_edges):
        blk = out[min(E, a):min(E, a + chunk_edges)]
        rng.standard_normal(blk.shape, dtype=np.float32, out=blk)
        blk *= scale
    return out


def make_graph(wl: Workload):
    """(senders, receivers, r) for a workload."""
    if wl.kind == "box":
        return periodic_box_graph(wl.N, wl.box, wl.cutoff)
    if wl.kind == "waterbox":
        s, rcv, r, _ = water_box_graph()
        return s, rcv, r
    s, rcv = poisson_graph(wl.N, wl.mean_degree)
    return s, rcv, random_edge_vectors(len(s))


# ---------------------------------------------------------------- water box

WATER_BOX = dict(n_atoms=1503, box=25.0, min_dist=0.9, cutoff=5.0, pad=0.10, C=128, L=3, hidden=64, n_bessel=8)


def random_sequential_packing(n_atoms: int, box: float, min_dist: float, seed: int = SEED_GRAPH):
    """Positions added one by one uniformly in a periodic cube, rejecting any
    closer than min_dist (minimum image) to an accepted one."""
    rng = np.random.default_rng(seed)
    pos = np.empty((n_atoms, 3))
    n = 0
    while n < n_atoms:
        cand = rng.uniform(0.0, box, size=(256, 3))
        for c in cand:
            if n:
                d = pos[:n] - c
                d -= box * np.round(d / box)
                if np.min(np.einsum("ij,ij->i", d, d)) < min_dist * min_dist:
                    continue
            pos[n] = c
            n += 1
            if n == n_atoms:
                break
    return pos


def padded_box_graph(pos: np.ndarray, box: float, cutoff: float, pad: float):
    """Ordered pairs (receiver i, sender j != i) within the cutoff (minimum
    image), r = pos[j] - pos[i], then int(E * pad) dummy edges i -> i
    (round-robin over atoms, r = (cutoff, 0, 0)); everything sorted by receiver,
    stable.  Returns (senders, receivers, r, is_dummy)."""
    n = len(pos)
    d = pos[None, :, :] - pos[:, None, :]
    d -= box * np.round(d / box)
    dist = np.linalg.norm(d, axis=-1)
    mask = (dist < cutoff) & ~np.eye(n, dtype=bool)
    recv, send = np.nonzero(mask)
    r = d[recv, send]
    n_pad = int(len(recv) * pad)
    dummy_nodes = np.arange(n_pad) % n
    recv = np.concatenate([recv, dummy_nodes])
    send = np.concatenate([send, dummy_nodes])
    r = np.concatenate([r, np.tile([[cutoff, 0.0, 0.0]], (n_pad, 1))])
    is_dummy = np.concatenate([np.zeros(len(recv) - n_pad, bool), np.ones(n_pad, bool)])
    order = np.argsort(recv, kind="stable")
    return (send[order].astype(np.int32), recv[order].astype(np.int32), r[order].astype(np.float32),
            is_dummy[order])


def radial_mlp_params(P: int, C: int, hidden: int = 64, n_bessel: int = 8, seed: int = SEED_W):
    """Seeded weights of the 2-hidden-layer radial MLP (n_bessel -> hidden ->
    hidden -> P*C, SiLU), fp32, Kaiming-style scaling."""
    rng = np.random.default_rng(seed)
    dims = [n_bessel, hidden, hidden, P * C]
    return [(rng.standard_normal((a, b)).astype(np.float32) / np.float32(np.sqrt(a))) for a, b in zip(dims[:-1], dims[1:])]


def radial_weights(r: np.ndarray, cutoff: float, params, P: int, C: int, is_dummy=None,
                   n_bessel: int = 8, p_env: int = 6) -> np.ndarray:
    """w[E, P, C] = envelope(d) * MLP(bessel(d)) for d = |r| (fp32): Bessel
    basis sqrt(2/rc) sin(n pi d / rc) / d, n = 1..n_bessel; polynomial envelope
    of order p_env (1 at d = 0, zero with its first two derivatives at the
    cutoff); dummy edges get w = 0."""
    d = np.linalg.norm(r.astype(np.float64), axis=1)
    u = np.clip(d / cutoff, 0.0, 1.0)
    p = p_env
    env = 1.0 - (p + 1) * (p + 2) / 2 * u ** p + p * (p + 2) * u ** (p + 1) - p * (p + 1) / 2 * u ** (p + 2)
    n = np.arange(1, n_bessel + 1)
    safe = np.maximum(d, 1e-9)
    bes = np.sqrt(2.0 / cutoff) * np.sin(n[None, :] * np.pi * d[:, None] / cutoff) / safe[:, None]
    silu = lambda z: z / (1.0 + np.exp(-z))
    h = bes.astype(np.float32)
    for i, W in enumerate(params):
        h = h @ W
        if i < len(params) - 1:
            h = silu(h).astype(np.float32)
    w = (h * env[:, None].astype(np.float32)).reshape(len(d), P, C).astype(np.float32)
    if is_dummy is not None:
        w[is_dummy] = 0.0
    return w


_WATER_GRAPH = None


def water_box_graph():
    """(senders, receivers, r, is_dummy) of the MACE(a)-shaped water box
    (WATER_BOX settings), built once per process."""
    global _WATER_GRAPH
    if _WATER_GRAPH is None:
        c = WATER_BOX
        pos = random_sequential_packing(c["n_atoms"], c["box"], c["min_dist"])
        _WATER_GRAPH = padded_box_graph(pos, c["box"], c["cutoff"], c["pad"])
    return _WATER_GRAPH


def water_box_system():
    """The water box as a function of positions: (pos [n][3] fp64, senders,
    receivers, shift [E][3] fp64, is_dummy) with r = pos[s] - pos[rcv] + shift
    for every edge (the minimum-image shift; (cutoff, 0, 0) on the dummy
    i -> i edges, whose r then does not depend on the positions)."""
    c = WATER_BOX
    pos = random_sequential_packing(c["n_atoms"], c["box"], c["min_dist"])
    s, rcv, r, is_dummy = water_box_graph()
    d = pos[s] - pos[rcv]
    shift = -c["box"] * np.round(d / c["box"])
    shift[is_dummy] = [c["cutoff"], 0.0, 0.0]
    return pos, s, rcv, shift, is_dummy


def water_box_weights(P: int, C: int) -> np.ndarray:
    """Radial weights w[E, P, C] of the water box's edges (zero on dummies)."""
    _, _, r, is_dummy = water_box_graph()
    params = radial_mlp_params(P, C, WATER_BOX["hidden"], WATER_BOX["n_bessel"])
    return radial_weights(r, WATER_BOX["cutoff"], params, P, C, is_dummy=is_dummy,
                          n_bessel=WATER_BOX["n_bessel"])


WORKLOADS["waterbox"] = Workload("waterbox", WATER_BOX["n_atoms"], WATER_BOX["C"], _natural(WATER_BOX["L"]),
                                 WATER_BOX["L"], _natural(WATER_BOX["L"]), "waterbox", box=WATER_BOX["box"],
                                 cutoff=WATER_BOX["cutoff"])
