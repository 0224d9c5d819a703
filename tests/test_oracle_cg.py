"""Pins for the oracle's Clebsch-Gordan coefficients (no GPU).

FlashCart (arXiv 2610.06409), App. B: an admissible path's coupling is unique
up to normalisation.  The oracle fixes the normalisation (orthonormal), the
phase (Condon-Shortley, Racah formula) and the real basis; these tests pin each
choice to something other than the oracle itself: a library routine (SymPy's
Wigner module), closed forms, orthogonality, and the Gaunt identity that ties
the real CG basis to the real harmonics.
"""
import itertools
from math import comb, sqrt

import numpy as np
import pytest

from oracle.cg import cg_complex, real_cg
from oracle.sh import sh

L_MAX = 3


def all_triples(lmax=L_MAX):
    for l1, l2, l3 in itertools.product(range(lmax + 1), repeat=3):
        if abs(l1 - l2) <= l3 <= l1 + l2:
            yield l1, l2, l3


def test_complex_cg_matches_sympy():
    from sympy.physics.wigner import clebsch_gordan
    for l1, l2, l3 in all_triples():
        for m1 in range(-l1, l1 + 1):
            for m2 in range(-l2, l2 + 1):
                m3 = m1 + m2
                if abs(m3) > l3:
                    continue
                ref = float(clebsch_gordan(l1, l2, l3, m1, m2, m3))
                assert abs(cg_complex(l1, m1, l2, m2, l3, m3) - ref) < 1e-14, (l1, m1, l2, m2, l3, m3)


def test_complex_cg_stretched_closed_form():
    # J = j1 + j2: <j1 m1 j2 m2|J M> = sqrt(C(2j1, j1+m1) C(2j2, j2+m2) / C(2J, J+M))
    for j1 in range(4):
        for j2 in range(4):
            J = j1 + j2
            for m1 in range(-j1, j1 + 1):
                for m2 in range(-j2, j2 + 1):
                    M = m1 + m2
                    ref = sqrt(comb(2 * j1, j1 + m1) * comb(2 * j2, j2 + m2) / comb(2 * J, J + M))
                    assert abs(cg_complex(j1, m1, j2, m2, J, M) - ref) < 1e-14


def test_complex_cg_singlet_closed_form():
    # <j m j -m|0 0> = (-1)^(j-m) / sqrt(2j+1)
    for j in range(5):
        for m in range(-j, j + 1):
            ref = (-1) ** (j - m) / sqrt(2 * j + 1)
            assert abs(cg_complex(j, m, j, -m, 0, 0) - ref) < 1e-14


def test_complex_cg_selection_rules():
    assert cg_complex(1, 1, 1, 1, 1, 1) == 0.0          # m1 + m2 != M
    assert cg_complex(1, 0, 1, 0, 3, 0) == 0.0          # triangle violated
    assert cg_complex(1, 0, 1, 0, 1, 0) == 0.0          # odd path with all m = 0


@pytest.mark.parametrize("l1,l2,l3", list(all_triples()))
def test_real_cg_orthonormal(l1, l2, l3):
    C = real_cg(l1, l2, l3)
    G = np.einsum("abk,abq->kq", C, C)
    assert np.max(np.abs(G - np.eye(2 * l3 + 1))) < 1e-13


@pytest.mark.parametrize("l1,l2,l3", list(all_triples()))
def test_real_cg_canonical_sign(l1, l2, l3):
    flat = real_cg(l1, l2, l3).reshape(-1)
    first = flat[np.nonzero(np.abs(flat) > 1e-9)[0][0]]
    assert first > 0


def test_real_cg_identity_paths():
    for l in range(L_MAX + 1):
        I = np.eye(2 * l + 1)
        assert np.max(np.abs(real_cg(l, 0, l)[:, 0, :] - I)) < 1e-14      # l x 0 -> l
        assert np.max(np.abs(real_cg(0, l, l)[0, :, :] - I)) < 1e-14      # 0 x l -> l
        # l x l -> 0 : delta_{m1 m2} / sqrt(2l+1) (canonical sign positive)
        assert np.max(np.abs(real_cg(l, l, 0)[:, :, 0] - I / np.sqrt(2 * l + 1))) < 1e-14


@pytest.mark.parametrize("l1,l2,l3", [t for t in all_triples() if sum(t) % 2 == 0])
def test_gaunt_identity_ties_cg_to_sh(l1, l2, l3):
    """sum_{m1 m2} C[m1,m2,m3] Y_l1m1(u) Y_l2m2(u) = kappa * Y_l3m3(u) with one
    kappa for every u and m3 (even paths): the real CG basis is the basis of
    the real harmonics.  |kappa| = sqrt((2l1+1)(2l2+1)/(2l3+1)) |<l1 0 l2 0|l3 0>|
    under component normalisation; its sign follows the canonical-sign rule."""
    rng = np.random.default_rng(7)
    u = rng.standard_normal((64, 3))
    Y = sh(u, L_MAX)
    Y1 = Y[:, l1 * l1:(l1 + 1) ** 2]
    Y2 = Y[:, l2 * l2:(l2 + 1) ** 2]
    Y3 = Y[:, l3 * l3:(l3 + 1) ** 2]
    lhs = np.einsum("abk,ea,eb->ek", real_cg(l1, l2, l3), Y1, Y2)
    expected = sqrt((2 * l1 + 1) * (2 * l2 + 1) / (2 * l3 + 1)) * abs(cg_complex(l1, 0, l2, 0, l3, 0))
    assert expected > 1e-3
    # one kappa for all u and m3; its sign follows the canonical-sign rule
    kappa = float((lhs * Y3).sum() / (Y3 * Y3).sum())
    assert abs(abs(kappa) - expected) < 1e-12
    assert np.max(np.abs(lhs - kappa * Y3)) < 1e-12


@pytest.mark.parametrize("l1,l2,l3", [t for t in all_triples() if sum(t) % 2 == 1])
def test_odd_paths_vanish_on_equal_arguments(l1, l2, l3):
    """Odd paths are antisymmetric couplings: contracting them with Y(u) Y(u)
    gives zero (their Gaunt coefficient <l1 0 l2 0|l3 0> vanishes)."""
    rng = np.random.default_rng(8)
    u = rng.standard_normal((16, 3))
    Y = sh(u, L_MAX)
    lhs = np.einsum("abk,ea,eb->ek", real_cg(l1, l2, l3), Y[:, l1 * l1:(l1 + 1) ** 2],
                    Y[:, l2 * l2:(l2 + 1) ** 2])
    assert np.max(np.abs(lhs)) < 1e-12
