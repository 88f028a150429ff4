"""Writes the regression fixtures in this folder from the CPU oracle only.

Run from the repository root: ``python tests/golden/make_golden.py``.
paley_h12.txt is the Paley construction I for q = 11 (quadratic residues
mod 11 are {1, 3, 4, 5, 9}); its algebraic checks (H H^T = 12 I, H = I + S
with S skew) live in tests/test_oracle_pins.py.  The fixture freezes the
sign pattern so that a later change to the construction is caught.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import oracle as O  # noqa: E402


def main():
    H = O.paley1(11)
    with open(os.path.join(HERE, "paley_h12.txt"), "w") as f:
        f.write("# Paley-I Hadamard of order 12 (q = 11), rows of H = I + S,\n")
        f.write("# S = [[0, 1^T], [-1, Q]], Q[i][j] = chi((j - i) mod 11).\n")
        f.write("# Written by tests/golden/make_golden.py from oracle/ only.\n")
        for row in H:
            f.write(" ".join("%2d" % v for v in row) + "\n")


if __name__ == "__main__":
    main()
