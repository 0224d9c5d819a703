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


def _natural(L: int) -> str:
    return "+".join(f"{l}{'e' if l % 2 == 0 else 'o'}" for l in range(L + 1))


WORKLOADS = {
    "tiny": Workload("tiny", 256, 32, "0e+1o", 2, _natural(2), "box"),
    "lmax2": Workload("lmax2", 32768, 128, _natural(2), 2, _natural(2), "poisson"),
    "lmax3": Workload("lmax3", 16384, 128, _natural(3), 3, _natural(3), "poisson"),
}
for _C in (64, 128, 256, 512, 1024):
    WORKLOADS[f"sweepC{_C}"] = Workload(f"sweepC{_C}", (1 << 22) // _C, _C, _natural(2), 2,
                                        _natural(2), "poisson")


def natural_irreps(L: int) -> str:
    """'0e+1o+...' up to L (natural parity)."""
    return _natural(L)


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
    s, rcv = poisson_graph(wl.N, wl.mean_degree)
    return s, rcv, random_edge_vectors(len(s))
