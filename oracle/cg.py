"""Clebsch-Gordan coefficients, complex and real basis (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

FlashCart (arXiv 2610.06409), App. B "Background": an admissible path obeys
the triangle inequalities and its equivariant bilinear coupling is unique up to
normalisation, so spherical and Cartesian products encode the same coupling.
The pages do not print the coefficients; the readings used here:

* complex CG <l1 m1 l2 m2 | l3 m3> by the Racah formula, evaluated as an exact
  rational under one final square root (Condon-Shortley phase);
* real basis by the unitary change of basis U^l (rows: real m, columns:
  complex mu), which maps Condon-Shortley complex harmonics onto the real
  harmonics of ``oracle/sh.py``:
      m > 0 : ((-1)^m |m> + |-m>) / sqrt2
      m = 0 : |0>
      m < 0 : i (|m> - (-1)^m |-m>) / sqrt2
  C[m1, m2, m3] = sum U3[m3, mu3] conj(U1[m1, mu1]) conj(U2[m2, mu2]) <..|..>.
  For l1 + l2 + l3 even the sum is real (checked); odd sums (both-parity
  variant, not used by the convolution) keep the imaginary part;
* canonical sign: the first entry with |c| > 1e-9 in (m1, m2, m3) order is
  made positive;
* no further normalisation: sum_{m1,m2} C[m1,m2,m3] C[m1,m2,m3'] = delta.
"""
from __future__ import annotations

from fractions import Fraction
from functools import lru_cache
from math import factorial, sqrt

import numpy as np


@lru_cache(maxsize=None)
def cg_complex(j1: int, m1: int, j2: int, m2: int, J: int, M: int) -> float:
    """<j1 m1 j2 m2 | J M> (integer j) by the Racah formula, exact until the
    final square root."""
    if m1 + m2 != M:
        return 0.0
    if not (abs(j1 - j2) <= J <= j1 + j2):
        return 0.0
    if abs(m1) > j1 or abs(m2) > j2 or abs(M) > J:
        return 0.0
    f = factorial
    pref2 = Fraction((2 * J + 1) * f(J + j1 - j2) * f(J - j1 + j2) * f(j1 + j2 - J),
                     f(j1 + j2 + J + 1))
    pref2 *= f(J + M) * f(J - M) * f(j1 - m1) * f(j1 + m1) * f(j2 - m2) * f(j2 + m2)
    s = Fraction(0)
    for k in range(0, j1 + j2 + J + 1):
        args = (k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k)
        if min(args) < 0:
            continue
        den = 1
        for a in args:
            den *= f(a)
        s += Fraction((-1) ** k, den)
    if s == 0:
        return 0.0
    val2 = pref2 * s * s
    # int / int true division is correctly rounded, so the only rounding
    # steps are that division and the square root.
    return (1.0 if s > 0 else -1.0) * sqrt(val2.numerator / val2.denominator)


def real_basis(l: int) -> np.ndarray:
    """U^l, (2l+1)x(2l+1) complex; row index m+l (real), column mu+l (complex)."""
    U = np.zeros((2 * l + 1, 2 * l + 1), dtype=np.complex128)
    r2 = 1.0 / np.sqrt(2.0)
    for m in range(-l, l + 1):
        if m > 0:
            U[m + l, m + l] = (-1) ** m * r2
            U[m + l, -m + l] = r2
        elif m == 0:
            U[l, l] = 1.0
        else:
            U[m + l, m + l] = 1j * r2
            U[m + l, -m + l] = -1j * (-1) ** m * r2
    return U


def complex_cg_tensor(l1: int, l2: int, l3: int) -> np.ndarray:
    T = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for a in range(-l1, l1 + 1):
        for b in range(-l2, l2 + 1):
            c = a + b
            if abs(c) <= l3:
                T[a + l1, b + l2, c + l3] = cg_complex(l1, a, l2, b, l3, c)
    return T


@lru_cache(maxsize=None)
def _real_cg_cached(l1: int, l2: int, l3: int) -> np.ndarray:
    T = complex_cg_tensor(l1, l2, l3)
    U1, U2, U3 = real_basis(l1), real_basis(l2), real_basis(l3)
    Cc = np.einsum("ia,jb,kc,abc->ijk", U1.conj(), U2.conj(), U3, T)
    if (l1 + l2 + l3) % 2 == 0:
        assert np.max(np.abs(Cc.imag)) < 1e-12, "even path must be real"
        C = Cc.real.copy()
    else:
        assert np.max(np.abs(Cc.real)) < 1e-12, "odd path must be imaginary"
        C = Cc.imag.copy()
    flat = C.reshape(-1)
    for v in flat:
        if abs(v) > 1e-9:
            if v < 0:
                C = -C
            break
    C[np.abs(C) < 1e-15] = 0.0
    C.setflags(write=False)
    return C


def real_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    """Real-basis coupling C[m1+l1, m2+l2, m3+l3] (fp64, read-only)."""
    return _real_cg_cached(l1, l2, l3)
