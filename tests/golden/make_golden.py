"""Writes the stored oracle values under tests/golden/.  Calls only oracle/.

No page prints a worked example or a coefficient table, so these files are
not the pages' numbers: they freeze the oracle's real-basis Clebsch-Gordan
table (FlashCart, arXiv 2610.06409, App. B: the admissible-path coupling,
unique up to normalisation; normalisation, phase and basis as read in
oracle/cg.py) so that any later change to it shows up as a test failure.

    python tests/golden/make_golden.py
"""
import itertools
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle.cg import real_cg  # noqa: E402


def main():
    lines = ["# real-basis CG, natural-parity paths l1,l2,l3 <= 3 (l1+l2+l3 even, triangle)",
             "# written by tests/golden/make_golden.py from oracle/cg.py",
             "# columns: l1 l2 l3 m1 m2 m3 value   (nonzero entries, |value| > 1e-15)"]
    for l1, l2, l3 in itertools.product(range(4), repeat=3):
        if abs(l1 - l2) <= l3 <= l1 + l2 and (l1 + l2 + l3) % 2 == 0:
            C = real_cg(l1, l2, l3)
            for a, b, c in itertools.product(range(2 * l1 + 1), range(2 * l2 + 1), range(2 * l3 + 1)):
                v = C[a, b, c]
                if abs(v) > 1e-15:
                    lines.append(f"{l1} {l2} {l3} {a - l1} {b - l2} {c - l3} {v:.17e}")
    with open(os.path.join(HERE, "real_cg_natural_l3.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
