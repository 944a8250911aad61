"""Sylvester Hadamard matrix (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"Fast Quantized Johnson - Lindenstrauss Transforms" builds both constructions
from randomized Hadamard transforms ("In short"; "The paper" abstract). The
oracle applies them as explicit matrices, not as a fast transform. Ordering
is Sylvester (natural) order: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]].
The normalised matrix H / sqrt(d) is orthogonal.
"""

import numpy as np


def sylvester(d):
    """Unnormalised d x d Hadamard matrix in Sylvester order (d a power of two)."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    H = np.ones((1, 1), dtype=np.float64)
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def normalised(d):
    """H / sqrt(d)."""
    return sylvester(d) / np.sqrt(d)
