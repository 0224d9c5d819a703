"""Symmetric contraction of correlation order 2 on the GPU against the oracle
(needs a B200): forward B and backward dA, dW1, dW2 for every (L_A, L_out)
shape class, several species, channel counts with a ragged tile and node
counts that do not fill the grid; out-of-range species flagged; the
backward bitwise reproducible."""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import binding as B
from equivariant_gnn_message_edge_b200.conv import SymmetricContraction
from equivariant_gnn_message_edge_b200.workloads import natural_irreps
from oracle import symcontract as sc
from tests.gpu_common import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _case(LA, Lout, C, N, S, seed):
    rng = np.random.default_rng(seed)
    P = len(sc.sym_paths(LA, Lout))
    A = rng.standard_normal((N, (LA + 1) ** 2, C)).astype(np.float32)
    z = rng.integers(0, S, size=N).astype(np.int32)
    W1 = rng.standard_normal((S, min(LA, Lout) + 1, C)).astype(np.float32)
    W2 = (rng.standard_normal((S, P, C)) / np.sqrt(P)).astype(np.float32)
    gB = rng.standard_normal((N, (Lout + 1) ** 2, C)).astype(np.float32)
    return A, z, W1, W2, gB


@pytest.mark.parametrize("LA,Lout,C,N,S", [(1, 1, 32, 50, 1), (2, 2, 64, 1000, 2), (2, 1, 132, 333, 3),
                                           (3, 3, 128, 700, 2), (3, 1, 64, 129, 5), (1, 3, 36, 77, 2),
                                           (2, 0, 32, 40, 16)])
def test_symmetric_contraction_matches_oracle(LA, Lout, C, N, S):
    A, z, W1, W2, gB = _case(LA, Lout, C, N, S, seed=LA * 10 + Lout + C)
    op = SymmetricContraction(natural_irreps(LA), natural_irreps(Lout), C, S)
    assert [tuple(p) for p in op.paths] == sc.sym_paths(LA, Lout)
    Bd = op.forward_raw(to_dev(A), to_dev(z), to_dev(W1), to_dev(W2))
    dA, dW1, dW2 = op.backward_raw(to_dev(A), to_dev(z), to_dev(W1), to_dev(W2), to_dev(gB))
    torch.cuda.synchronize()
    assert B.eqconv_get_device_error(op.plan) == B.EQCONV_OK
    assert_close("B", Bd.cpu().numpy(), sc.forward(A, z, W1, W2, LA, Lout))
    dAr, dW1r, dW2r = sc.backward(A, z, W1, W2, gB, LA, Lout, S)
    assert_close("dA", dA.cpu().numpy(), dAr)
    assert_close("dW1", dW1.cpu().numpy(), dW1r)
    assert_close("dW2", dW2.cpu().numpy(), dW2r)


def test_symmetric_contraction_autograd_and_determinism():
    LA, Lout, C, N, S = 2, 1, 64, 900, 2
    A, z, W1, W2, gB = _case(LA, Lout, C, N, S, seed=7)
    op = SymmetricContraction(natural_irreps(LA), natural_irreps(Lout), C, S)
    Ad, W1d, W2d = (to_dev(t).requires_grad_(True) for t in (A, W1, W2))
    out = op(Ad, to_dev(z), W1d, W2d)
    g = torch.autograd.grad(out, [Ad, W1d, W2d], to_dev(gB))
    g2 = op.backward_raw(to_dev(A), to_dev(z), to_dev(W1), to_dev(W2), to_dev(gB))
    for a, b in zip(g, g2):
        assert torch.equal(a, b)


def test_out_of_range_species_is_flagged():
    LA, Lout, C, N, S = 1, 1, 32, 20, 2
    A, z, W1, W2, _ = _case(LA, Lout, C, N, S, seed=3)
    z[5] = 7
    op = SymmetricContraction(natural_irreps(LA), natural_irreps(Lout), C, S)
    Bd = op.forward_raw(to_dev(A), to_dev(z), to_dev(W1), to_dev(W2))
    torch.cuda.synchronize()
    assert B.eqconv_get_device_error(op.plan) == B.EQCONV_ERR_DEVICE_CHECK
    assert np.all(Bd.cpu().numpy()[5] == 0.0)
