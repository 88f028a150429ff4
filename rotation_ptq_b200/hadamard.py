"""Small Hadamard factor passed to ``rotate_quant`` as ``had_small``.

The 12,288-wide R4 rotation of Qwen3-8B's MLP ("SpinQuant, Reproduced",
section Q5) is H12 (x) H1024.  H1024 is the Sylvester matrix the kernels apply
as butterflies; H12 is not a power of two, so the caller hands the kernels its
12 x 12 sign pattern.  This module builds the Paley-I construction: for the
prime q = 11 (q = 3 mod 4), with chi the quadratic character mod q,
Q[i][j] = chi(j - i), S = [[0, 1^T], [-1, Q]], H12 = I + S.
"""
from __future__ import annotations

import numpy as np


def _legendre(r: int, q: int) -> int:
    r %= q
    if r == 0:
        return 0
    # Euler's criterion: r^((q-1)/2) = 1 (mod q) for quadratic residues
    return 1 if pow(r, (q - 1) // 2, q) == 1 else -1


def paley_h12() -> np.ndarray:
    """The 12 x 12 Paley-I Hadamard matrix as int8 (+-1), row-major."""
    q = 11
    h = np.eye(q + 1, dtype=np.int8)
    h[0, 1:] += 1
    h[1:, 0] -= 1
    for i in range(q):
        for j in range(q):
            h[i + 1, j + 1] += _legendre(j - i, q)
    return h
