"""Pins of the causal prefill oracle (CPU).

Row i equals the decode attention of query i over keys 0..i (brute force). The
first row returns the first value, and every row's weights sum to one with no
weight on later keys.
"""

import numpy as np

from oracle import attention


def test_rows_equal_decode_over_the_prefix():
    rng = np.random.default_rng(1)
    G, L, d = 2, 9, 8
    est = rng.standard_normal((G, L, L)) * 3
    v = rng.standard_normal((G, L, d))
    out, p = attention.prefill_attention(est, v, 0.7)
    for g in range(G):
        for i in range(L):
            w = np.exp(0.7 * est[g, i, :i + 1] - (0.7 * est[g, i, :i + 1]).max())
            w /= w.sum()
            assert np.allclose(out[g, i], w @ v[g, :i + 1], rtol=1e-13, atol=1e-13)
            assert np.allclose(p[g, i, :i + 1], w, rtol=1e-13) and not p[g, i, i + 1:].any()
    assert np.allclose(out[:, 0], v[:, 0], rtol=1e-14)
