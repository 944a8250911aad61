"""Pins for the oracle's 2-bit per-token values and decode attention.

KIVI abstract ("Vladimir Braverman" page): values are quantised per token to
2 bits, asymmetrically (zero point and scale). The pins: codes are the
nearest of the four levels z + c*s by brute force (ties either way);
|v - v_hat| <= s/2; constant groups; the packing order. For attention: scipy's
softmax; brute-force loops on tiny inputs; one key; equal scores; and
shift invariance.
"""

import numpy as np
import pytest
import scipy.special

from oracle import attention, kivi


def _vals(n, d, seed=0):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((n, d)).astype(np.float32)
    # snap to bf16 like the decode workload
    return (v.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)


def test_codes_are_nearest_level_brute_force():
    V = _vals(40, 64)
    words, scale, zero = kivi.quantize_values_2bit(V)
    codes = kivi.unpack_codes(words, 64)
    for n in range(40):
        for c in range(64):
            g = c // 32
            s, z = float(scale[n, g]), float(zero[n, g])
            dist = [abs(float(V[n, c]) - (z + lvl * s)) for lvl in range(4)]
            best = int(np.argmin(dist))
            if codes[n, c] != best:
                # only an (almost) exact tie may go either way
                assert abs(dist[codes[n, c]] - dist[best]) <= 1e-5 * s


def test_error_bound_and_levels():
    V = _vals(200, 128, seed=1)
    words, scale, zero = kivi.quantize_values_2bit(V)
    vhat = kivi.dequantize_values(words, scale, zero, 128)
    s = np.repeat(scale.astype(np.float64), 32, axis=1)
    z = np.repeat(zero.astype(np.float64), 32, axis=1)
    # fp16 rounding of z and s moves the grid by at most a few fp16 ulps
    slack = 3 * (np.abs(z) + 3 * s) * 2.0 ** -11
    assert np.all(np.abs(V - vhat) <= s / 2 + slack)
    mn = V.reshape(200, 4, 32).min(axis=2)
    assert np.array_equal(zero, mn.astype(np.float16))


def test_constant_group_and_packing():
    V = np.zeros((2, 32), dtype=np.float32)
    V[0, :] = 1.5
    V[1, :] = -0.25
    words, scale, zero = kivi.quantize_values_2bit(V)
    assert np.all(scale == 0) and np.all(words == 0)
    assert np.array_equal(kivi.dequantize_values(words, scale, zero, 32), V.astype(np.float64))
    # ramp of the four levels: code c at bits 2*(c % 16) of word c // 16
    ramp = np.tile(np.array([0.0, 1.0, 2.0, 3.0], dtype=np.float32), 8)[None, :]
    words, scale, zero = kivi.quantize_values_2bit(ramp)
    assert float(scale[0, 0]) == 1.0 and float(zero[0, 0]) == 0.0
    for c in range(32):
        assert (int(words[0, c // 16]) >> (2 * (c % 16))) & 3 == c % 4


def test_softmax_matches_scipy():
    x = np.random.default_rng(3).standard_normal((4, 7)) * 5
    assert np.allclose(attention.softmax(x), scipy.special.softmax(x, axis=-1), rtol=1e-14)


def test_decode_attention_brute_force():
    rng = np.random.default_rng(4)
    G, J, N, d = 2, 3, 6, 5
    est = rng.standard_normal((G, J, N)) * 3
    v = rng.standard_normal((G, N, d))
    out = attention.decode_attention(est, v, 0.7)
    for g in range(G):
        for j in range(J):
            w = [np.exp(0.7 * est[g, j, n]) for n in range(N)]
            tot = sum(w)
            for c in range(d):
                want = sum(w[n] * v[g, n, c] for n in range(N)) / tot
                assert abs(out[g, j, c] - want) < 1e-12


def test_attention_special_cases():
    rng = np.random.default_rng(5)
    v = rng.standard_normal((1, 4, 8))
    one = attention.decode_attention(np.array([[[2.0]]]), v[:, :1], 1.0)
    assert np.allclose(one[0, 0], v[0, 0])
    eq = attention.decode_attention(np.zeros((1, 1, 4)), v, 1.0)
    assert np.allclose(eq[0, 0], v[0].mean(axis=0))
    est = rng.standard_normal((1, 1, 4))
    assert np.allclose(attention.decode_attention(est, v, 1.0),
                       attention.decode_attention(est + 100.0, v, 1.0))
