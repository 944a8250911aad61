"""Pins of the KIVI per-channel key quantiser (oracle, CPU).

Brute force on tiny inputs, the reconstruction bound |k - k_hat| <= s/2 (plus
the fp16 rounding of the zero), constant channels, ragged token blocks, and
scores that equal a hand-written triple loop over the dequantised keys.
"""

import numpy as np

from oracle import kivi


def _brute(K):
    G, N, d = K.shape
    nb = (N + 31) // 32
    codes = np.zeros((G, N, d), dtype=np.int64)
    S = np.zeros((G, nb, d)); Z = np.zeros((G, nb, d))
    for g in range(G):
        for b in range(nb):
            for c in range(d):
                col = K[g, b * 32:(b + 1) * 32, c].astype(np.float32)
                z = np.float16(col.min())
                s = np.float16(np.float32((np.float32(col.max()) - np.float32(col.min())) / np.float32(3)))
                S[g, b, c], Z[g, b, c] = s, z
                for i, v in enumerate(col):
                    if np.float32(s) == 0:
                        q = 0
                    else:
                        t = np.float32(np.float32(v - np.float32(z)) / np.float32(s))
                        q = int(min(max(np.rint(t), 0), 3))
                    codes[g, b * 32 + i, c] = q
    return codes, S, Z


def test_brute_force_small():
    rng = np.random.default_rng(1)
    K = (rng.standard_normal((2, 45, 32)) * 3).astype(np.float32)       # a ragged second block of 13
    w, s, z = kivi.quantize_keys_per_channel(K)
    codes, S, Z = _brute(K)
    got = kivi.unpack_codes(w.reshape(-1, 2), 32).reshape(2, 45, 32)
    assert np.array_equal(got, codes)
    assert np.array_equal(s.astype(np.float64), S) and np.array_equal(z.astype(np.float64), Z)


def test_reconstruction_bound_and_constant_channel():
    rng = np.random.default_rng(2)
    K = rng.standard_normal((3, 64, 64)).astype(np.float32)
    K[1, :32, 5] = 0.75                                                  # a constant channel block
    w, s, z = kivi.quantize_keys_per_channel(K)
    khat = kivi.dequantize_keys_per_channel(w, s, z)
    blk = np.arange(64) // 32
    S = s.astype(np.float64)[:, blk, :]
    Zerr = np.abs(z.astype(np.float64) - K.reshape(3, 2, 32, 64).min(axis=2))[:, blk, :]
    assert np.all(np.abs(K - khat) <= S / 2 + Zerr + 1e-6 * np.abs(K) + 1e-9)
    assert np.all(khat[1, :32, 5] == np.float16(0.75))


def test_key_scores_loop():
    rng = np.random.default_rng(3)
    K = rng.standard_normal((2, 40, 32)).astype(np.float32)
    Q = rng.standard_normal((2, 3, 32))
    w, s, z = kivi.quantize_keys_per_channel(K)
    got = kivi.key_scores(w, s, z, Q)
    codes = kivi.unpack_codes(w.reshape(-1, 2), 32).reshape(2, 40, 32)
    for g in range(2):
        for j in range(3):
            for n in range(40):
                b = n // 32
                want = sum(Q[g, j, c] * (codes[g, n, c] * float(s[g, b, c]) + float(z[g, b, c])) for c in range(32))
                assert abs(got[g, j, n] - want) <= 1e-12 * (1 + abs(want))
