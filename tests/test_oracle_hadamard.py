"""Pins for the oracle's Sylvester Hadamard matrix.

"Fast Quantized Johnson - Lindenstrauss Transforms" ("In short", "The paper"
abstract) builds both constructions from randomized Hadamard transforms.
The pins: scipy's Hadamard routine; the closed form H[i][j] = (-1)^popcount(i & j)
by brute force; H H = d I; and the normalised matrix is an isometry.
"""

import numpy as np
import pytest
import scipy.linalg

from oracle import hadamard


@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_matches_scipy_sylvester(d):
    assert np.array_equal(hadamard.sylvester(d), scipy.linalg.hadamard(d).astype(np.float64))


@pytest.mark.parametrize("d", [1, 2, 4, 8, 16])
def test_popcount_closed_form_brute_force(d):
    H = hadamard.sylvester(d)
    for i in range(d):
        for j in range(d):
            assert H[i][j] == (-1) ** bin(i & j).count("1")


@pytest.mark.parametrize("d", [2, 16, 128])
def test_orthogonality_and_isometry(d):
    H = hadamard.sylvester(d)
    assert np.array_equal(H @ H, d * np.eye(d))
    x = np.random.default_rng(d).standard_normal((5, d))
    Hn = hadamard.normalised(d)
    assert np.allclose(np.linalg.norm(x @ Hn.T, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


@pytest.mark.parametrize("d", [0, 3, 6, 12])
def test_rejects_non_power_of_two(d):
    with pytest.raises(ValueError):
        hadamard.sylvester(d)
