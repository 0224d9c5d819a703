"""Symmetric contraction of correlation order 2 (MACE product basis), forward
and backward (oracle).

Test infrastructure only (see ``oracle/__init__.py``).

e3j (arXiv 2609.35099), abstract and Table 3: the MACE(a) model's product
basis has correlation order 2 and its tensor products are the operation the
page measures at over 80% of the GPU's memory bandwidth.  FlashCart (arXiv
2610.06409) §5 and App. B: the correlation ladder builds higher-order
features at each atom from repeated channel-diagonal products of the atom's
own features along the admissible paths, with learned weights per path and
channel; App. D: weights per element (species).

Reading (the pages print no formula): for node i of species z_i with features
A[i] (irreps a natural-parity prefix 0e+1o+... up to L_A, C channels each),

    B[i, L M, c] =  W1[z_i, L, c] A[i, L M, c]                                      (order 1, L <= L_A)
                 +  sum_{q = (l1, l2, L)} W2[z_i, q, c] sum_{m1, m2} C_q[m1, m2, M] A[i, l1 m1, c] A[i, l2 m2, c]

with q over l1 <= l2 <= L_A, L <= L_out, |l1 - l2| <= L <= l1 + l2 and
l1 + l2 + L even (natural parity; the odd couplings of equal inputs vanish,
and (l2, l1, L) equals (l1, l2, L) on the symmetric product, so each
unordered pair appears once), ordered by (l1, l2, L).  C_q is the real CG of
``oracle/cg.py``.  Backward given gB:

    dA[i, l m, c]  = W1[z_i, l, c] gB[i, l m, c]
                   + sum_q W2[z_i, q, c] ( [l1 = l] sum_{m2, M} C_q[m, m2, M] A[l2 m2] gB[L M]
                                          + [l2 = l] sum_{m1, M} C_q[m1, m, M] A[l1 m1] gB[L M] )
    dW1[s, L, c]   = sum_{i: z_i = s} sum_M A[i, L M, c] gB[i, L M, c]
    dW2[s, q, c]   = sum_{i: z_i = s} sum_{m1, m2, M} C_q A A gB

NumPy einsum, fp64.
"""
from __future__ import annotations

import numpy as np

from .cg import real_cg


def sym_paths(L_A: int, L_out: int) -> list[tuple[int, int, int]]:
    """The order-2 paths (l1, l2, L), ordered by (l1, l2, L)."""
    out = []
    for l1 in range(L_A + 1):
        for l2 in range(l1, L_A + 1):
            for L in range(L_out + 1):
                if abs(l1 - l2) <= L <= l1 + l2 and (l1 + l2 + L) % 2 == 0:
                    out.append((l1, l2, L))
    return out


def _blk(A, l):
    return A[:, l * l:(l + 1) * (l + 1), :]


def forward(A, species, W1, W2, L_A: int, L_out: int) -> np.ndarray:
    """B [N][(L_out+1)^2][C]; W1 [S][min(L_A, L_out)+1][C], W2 [S][P][C]."""
    A = np.asarray(A, dtype=np.float64)
    z = np.asarray(species)
    W1, W2 = np.asarray(W1, dtype=np.float64)[z], np.asarray(W2, dtype=np.float64)[z]   # per node
    N, _, C = A.shape
    B = np.zeros((N, (L_out + 1) ** 2, C))
    for L in range(min(L_A, L_out) + 1):
        B[:, L * L:(L + 1) ** 2, :] += W1[:, L, None, :] * _blk(A, L)
    for q, (l1, l2, L) in enumerate(sym_paths(L_A, L_out)):
        t = np.einsum("abk,nac,nbc->nkc", real_cg(l1, l2, L), _blk(A, l1), _blk(A, l2))
        B[:, L * L:(L + 1) ** 2, :] += W2[:, q, None, :] * t
    return B


def backward(A, species, W1, W2, gB, L_A: int, L_out: int, n_species: int):
    """(dA, dW1, dW2)."""
    A, gB = np.asarray(A, dtype=np.float64), np.asarray(gB, dtype=np.float64)
    z = np.asarray(species)
    W1n, W2n = np.asarray(W1, dtype=np.float64)[z], np.asarray(W2, dtype=np.float64)[z]
    N, _, C = A.shape
    paths = sym_paths(L_A, L_out)
    dA = np.zeros_like(A)
    dW1 = np.zeros((n_species, min(L_A, L_out) + 1, C))
    dW2 = np.zeros((n_species, len(paths), C))
    for L in range(min(L_A, L_out) + 1):
        g = _blk(gB, L)
        dA[:, L * L:(L + 1) ** 2, :] += W1n[:, L, None, :] * g
        np.add.at(dW1[:, L, :], z, np.einsum("nmc,nmc->nc", _blk(A, L), g))
    for q, (l1, l2, L) in enumerate(paths):
        Cq = real_cg(l1, l2, L)
        a1, a2, g = _blk(A, l1), _blk(A, l2), _blk(gB, L)
        w = W2n[:, q, None, :]
        dA[:, l1 * l1:(l1 + 1) ** 2, :] += w * np.einsum("abk,nbc,nkc->nac", Cq, a2, g)
        dA[:, l2 * l2:(l2 + 1) ** 2, :] += w * np.einsum("abk,nac,nkc->nbc", Cq, a1, g)
        np.add.at(dW2[:, q, :], z, np.einsum("abk,nac,nbc,nkc->nc", Cq, a1, a2, g))
    return dA, dW1, dW2
