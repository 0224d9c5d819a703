"""Pins for the oracle's symmetric contraction of correlation order 2 (no GPU).

e3j (arXiv 2609.35099) Table 3: MACE(a) with correlation order 2; FlashCart
(arXiv 2610.06409) §5 / App. B: the node-local correlation ladder.  What pins
the oracle, independently of its own formula:
* on one species its order-2 term equals the (independently pinned)
  node-local product u (x) v with u = v = A and the weights of each unordered
  pair placed on the ordered pair (l1 <= l2), zero on the other;
* rotation equivariance (Wigner matrices from the harmonics) and the
  inversion signs (-1)^L of the outputs;
* the order-1 term alone is the per-irrep scaling W1 A (closed form);
* a node's output depends on its own species' weights only;
* the backward: B is quadratic in A, so central differences are exact, and
  <gB, dB/dA . V> = <dA, V>; B is linear in the weights, so
  <dW1, W1> + <dW2, W2> = <gB, B>; homogeneity gives
  <dA, A> = <gB, B1> + 2 <gB, B2>;
* planted mistakes (one factor of the product dropped from dA, a species
  mix-up, a sign flip) fail these pins.
"""
import numpy as np
import pytest

from equivariant_gnn_message_edge_b200.workloads import natural_irreps
from oracle import conv
from oracle import symcontract as sc
from oracle.cg import real_cg
from oracle.nodeprod import node_product
from tests.helpers import block_wigner, parity_signs, random_rotation

CASES = [(1, 1), (2, 2), (3, 3), (2, 3), (3, 1), (1, 2)]


def _setup(LA, Lout, C=4, N=9, S=3, seed=0):
    rng = np.random.default_rng(seed)
    P = len(sc.sym_paths(LA, Lout))
    A = rng.standard_normal((N, (LA + 1) ** 2, C))
    z = rng.integers(0, S, size=N)
    W1 = rng.standard_normal((S, min(LA, Lout) + 1, C))
    W2 = rng.standard_normal((S, P, C))
    gB = rng.standard_normal((N, (Lout + 1) ** 2, C))
    return A, z, W1, W2, gB


def test_path_list():
    assert sc.sym_paths(2, 2) == [(0, 0, 0), (0, 1, 1), (0, 2, 2), (1, 1, 0), (1, 1, 2), (1, 2, 1), (2, 2, 0),
                                  (2, 2, 2)]
    for LA, Lout in CASES:
        for l1, l2, L in sc.sym_paths(LA, Lout):
            assert l1 <= l2 and (l1 + l2 + L) % 2 == 0 and abs(l1 - l2) <= L <= l1 + l2
            if l1 == l2:   # the coupling of two equal inputs is symmetric in (m1, m2)
                Cq = real_cg(l1, l2, L)
                assert np.max(np.abs(Cq - Cq.transpose(1, 0, 2))) < 1e-13


@pytest.mark.parametrize("LA,Lout", CASES)
def test_order2_term_is_the_node_product_of_A_with_itself(LA, Lout):
    A, _, _, W2, _ = _setup(LA, Lout, S=1)
    z = np.zeros(A.shape[0], int)
    W1 = np.zeros((1, min(LA, Lout) + 1, A.shape[2]))
    prob = conv.Problem(natural_irreps(LA), LA, natural_irreps(Lout), A.shape[2])
    paths = sc.sym_paths(LA, Lout)
    w = np.zeros((prob.P, A.shape[2]))
    for p, q in enumerate(prob.paths):
        key = (q["l1"], q["l2"], q["l3"])
        if key in paths:
            w[p] = W2[0, paths.index(key)]
    got = sc.forward(A, z, W1, W2, LA, Lout)
    want = node_product(prob, A, A, w)
    assert np.max(np.abs(got - want)) < 1e-12 * max(1.0, np.max(np.abs(want)))


@pytest.mark.parametrize("LA,Lout", CASES)
def test_equivariance_and_parity(LA, Lout):
    A, z, W1, W2, _ = _setup(LA, Lout, seed=2)
    ins, outs = natural_irreps(LA), natural_irreps(Lout)
    for seed in range(3):
        R = random_rotation(seed)
        Din, Dout = block_wigner(R, ins), block_wigner(R, outs)
        rotA = np.einsum("ij,njc->nic", Din, A)
        got = sc.forward(rotA, z, W1, W2, LA, Lout)
        want = np.einsum("ij,njc->nic", Dout, sc.forward(A, z, W1, W2, LA, Lout))
        assert np.max(np.abs(got - want)) < 1e-9 * max(1.0, np.max(np.abs(want)))
    # inversion: A_l -> (-1)^l A_l gives B_L -> (-1)^L B_L
    sA, sB = parity_signs(ins), parity_signs(outs)
    got = sc.forward(sA[None, :, None] * A, z, W1, W2, LA, Lout)
    want = sB[None, :, None] * sc.forward(A, z, W1, W2, LA, Lout)
    assert np.max(np.abs(got - want)) < 1e-12 * max(1.0, np.max(np.abs(want)))


def test_order1_term_closed_form_and_species_selection():
    LA, Lout = 2, 2
    A, z, W1, W2, _ = _setup(LA, Lout, seed=3)
    B = sc.forward(A, z, W1, np.zeros_like(W2), LA, Lout)
    reps = np.repeat(W1[z], [1, 3, 5], axis=1)
    assert np.max(np.abs(B - reps * A)) < 1e-13
    # each node sees its own species' weights: nodes computed species by species agree
    full = sc.forward(A, z, W1, W2, LA, Lout)
    for s in range(W1.shape[0]):
        m = z == s
        if m.any():
            part = sc.forward(A[m], np.zeros(m.sum(), int), W1[s:s + 1], W2[s:s + 1], LA, Lout)
            assert np.max(np.abs(part - full[m])) < 1e-13


@pytest.mark.parametrize("LA,Lout", CASES)
def test_backward_exact_derivatives_and_identities(LA, Lout):
    A, z, W1, W2, gB = _setup(LA, Lout, seed=4)
    S = W1.shape[0]
    dA, dW1, dW2 = sc.backward(A, z, W1, W2, gB, LA, Lout, S)
    rng = np.random.default_rng(9)
    V = rng.standard_normal(A.shape)
    t = 0.5
    dirder = (sc.forward(A + t * V, z, W1, W2, LA, Lout) - sc.forward(A - t * V, z, W1, W2, LA, Lout)) / (2 * t)
    lhs, rhs = np.sum(gB * dirder), np.sum(dA * V)
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs))
    B = sc.forward(A, z, W1, W2, LA, Lout)
    assert abs(np.sum(dW1 * W1) + np.sum(dW2 * W2) - np.sum(gB * B)) < 1e-10 * max(1.0, abs(np.sum(gB * B)))
    B1 = sc.forward(A, z, W1, np.zeros_like(W2), LA, Lout)
    B2 = B - B1
    assert abs(np.sum(dA * A) - np.sum(gB * B1) - 2 * np.sum(gB * B2)) < 1e-10 * max(1.0, abs(np.sum(gB * B)))
    # weight gradients: B is linear in the weights, so central differences are exact too
    for Wi, dWi, k in ((W1, dW1, 1), (W2, dW2, 2)):
        U = rng.standard_normal(Wi.shape)
        args = lambda s: (W1 + s * U, W2) if k == 1 else (W1, W2 + s * U)
        d = (sc.forward(A, z, *args(t), LA, Lout) - sc.forward(A, z, *args(-t), LA, Lout)) / (2 * t)
        assert abs(np.sum(gB * d) - np.sum(dWi * U)) < 1e-10 * max(1.0, abs(np.sum(gB * d)))


def test_planted_mistakes_fail_the_pins(monkeypatch):
    LA, Lout = 2, 2
    A, z, W1, W2, gB = _setup(LA, Lout, seed=5)
    S = W1.shape[0]
    rng = np.random.default_rng(11)
    V = rng.standard_normal(A.shape)
    t = 0.5

    def vjp_gap(backward):
        dA, _, _ = backward(A, z, W1, W2, gB, LA, Lout, S)
        dirder = (sc.forward(A + t * V, z, W1, W2, LA, Lout) - sc.forward(A - t * V, z, W1, W2, LA, Lout)) / (2 * t)
        return abs(np.sum(gB * dirder) - np.sum(dA * V))

    assert vjp_gap(sc.backward) < 1e-9
    # (1) only the first factor's term in dA
    orig_einsum = np.einsum

    def one_factor(A_, z_, W1_, W2_, gB_, LA_, Lout_, S_):
        dA, dW1, dW2 = sc.backward(A_, z_, W1_, W2_, gB_, LA_, Lout_, S_)
        for q, (l1, l2, L) in enumerate(sc.sym_paths(LA_, Lout_)):
            a1, g = A_[:, l1 * l1:(l1 + 1) ** 2], gB_[:, L * L:(L + 1) ** 2]
            w = np.asarray(W2_)[z_][:, q, None, :]
            dA[:, l2 * l2:(l2 + 1) ** 2] -= w * orig_einsum("abk,nac,nkc->nbc", real_cg(l1, l2, L), a1, g)
        return dA, dW1, dW2

    assert vjp_gap(one_factor) > 1e-3
    # (2) species mix-up: every node takes species 0's weights
    B = sc.forward(A, z, W1, W2, LA, Lout)
    mixed = sc.forward(A, np.zeros_like(z), W1, W2, LA, Lout)
    m = z != 0
    assert m.any() and np.max(np.abs(mixed[m] - B[m])) > 1e-3
    # (3) a sign flip of one path breaks equality with the node product
    flipped = sc.forward(A, z, W1, W2 * np.where(np.arange(W2.shape[1]) == 4, -1.0, 1.0)[None, :, None], LA, Lout)
    assert np.max(np.abs(flipped - B)) > 1e-3
