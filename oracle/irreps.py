"""Irreps strings, block offsets and coupling paths (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

A feature row holds one block of 2l+1 components per irrep, each component a
run of C channels (FlashCart, App. D "Executing Cartesian tensor products",
Figure D1: rank blocks contiguous, components then channels within a block).
Every irrep carries the same C channels, so the product is channelwise
(FlashCart §5 and App. D: channel-diagonal products).

Paths (l1, l2, l3): l1 an input irrep, l2 a spherical-harmonic degree
0..L_sh with parity (-1)^l2, l3 an output irrep; admissible when
|l1-l2| <= l3 <= l1+l2 and p1 * (-1)^l2 == p3 (FlashCart App. B: triangle
inequalities; parity).  Reading: paths are ordered lexicographically by
(l1, l2, l3) and contributions of paths landing on the same output irrep are
summed.
"""
from __future__ import annotations

import re

_TOKEN = re.compile(r"^\s*(?:(\d+)x)?(\d+)([eo])\s*$")


def parse_irreps(s: str) -> list[tuple[int, int]]:
    """'0e+1o+2e' -> [(0, +1), (1, -1), (2, +1)].  A leading 'Nx' multiplicity
    is accepted only as '1x' (the channel count C is the multiplicity)."""
    out = []
    for tok in s.split("+"):
        m = _TOKEN.match(tok)
        if m is None:
            raise ValueError(f"bad irrep token {tok!r} in {s!r}")
        mult, l, p = m.groups()
        if mult is not None and int(mult) != 1:
            raise ValueError("multiplicity other than 1 is not supported (C is the multiplicity)")
        out.append((int(l), 1 if p == "e" else -1))
    return out


def block_offsets(irreps: list[tuple[int, int]]) -> tuple[list[int], int]:
    """Offsets of each irrep block inside a row, and the row length D."""
    offs, d = [], 0
    for l, _ in irreps:
        offs.append(d)
        d += 2 * l + 1
    return offs, d


def enumerate_paths(irreps_in, L_sh: int, irreps_out) -> list[dict]:
    """All admissible (l1, l2, l3) paths, ordered by (l1, l2, l3)."""
    ins = parse_irreps(irreps_in) if isinstance(irreps_in, str) else irreps_in
    outs = parse_irreps(irreps_out) if isinstance(irreps_out, str) else irreps_out
    off_in, _ = block_offsets(ins)
    off_out, _ = block_offsets(outs)
    paths = []
    for i1, (l1, p1) in enumerate(ins):
        for l2 in range(L_sh + 1):
            p2 = 1 if l2 % 2 == 0 else -1
            for i3, (l3, p3) in enumerate(outs):
                if abs(l1 - l2) <= l3 <= l1 + l2 and p1 * p2 == p3:
                    paths.append(dict(l1=l1, l2=l2, l3=l3, i1=i1, i3=i3,
                                      off1=off_in[i1], off2=l2 * l2, off3=off_out[i3]))
    paths.sort(key=lambda q: (q["l1"], q["l2"], q["l3"], q["i1"], q["i3"]))
    return paths
