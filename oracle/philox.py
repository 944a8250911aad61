"""Philox4x32-10 counter-based generator, uniforms and Box-Muller (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages draw the JL map S, the Hadamard diagonals and the dither at random.
They fix no generator: QJL abstract ("Majid Daliri" page) and "Fast Quantized
Johnson - Lindenstrauss Transforms", "Key concepts". Both the library and this
oracle must derive the same numbers from a seed, so each side implements the
same published generator independently. That generator is Philox4x32 with 10
rounds, from Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy
as 1, 2, 3" (SC'11):

    round:  (c0, c1, c2, c3) -> (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2),
                                 hi(M0*c0) ^ c3 ^ k1, lo(M0*c0))
    key schedule between rounds: k0 += W0, k1 += W1 (mod 2^32)
    M0 = 0xD2511F53, M1 = 0xCD9E8D57, W0 = 0x9E3779B9, W1 = 0xBB67AE85

Everything is vectorised over numpy uint64 arrays that hold 32-bit values.

Pins: the known-answer vectors published with the definition (three
(counter, key) inputs and their outputs) fix the bit stream. The tests also pin
the statistics (uniformity, Gaussian moments, permutation uniformity), and
they check that this generator and the library's own copy agree bit for bit.
"""

import numpy as np

M0 = 0xD2511F53
M1 = 0xCD9E8D57
W0 = 0x9E3779B9
W1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF

# Counter word 3 selects an independent stream per kind of random number.
STREAM_GAUSS = 0       # dense S entries, Gaussian diagonal D_g
STREAM_RADEMACHER = 1  # Rademacher diagonal D_r
STREAM_PERM = 2        # Fisher-Yates draws for the permutation Pi
STREAM_DITHER = 3      # D-FQJL dither, one block per (token, 8 coordinates)


def _u32(x):
    return np.asarray(x, dtype=np.uint64) & np.uint64(MASK32)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32-10 block function on broadcastable arrays of 32-bit words.

    Returns the four output words as uint64 arrays holding 32-bit values.
    """
    c0, c1, c2, c3 = _u32(c0), _u32(c1), _u32(c2), _u32(c3)
    k0 = np.broadcast_to(_u32(k0), np.broadcast(c0, c1, c2, c3).shape).copy()
    k1 = np.broadcast_to(_u32(k1), k0.shape).copy()
    m0, m1 = np.uint64(M0), np.uint64(M1)
    mask = np.uint64(MASK32)
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(W0)) & mask
            k1 = (k1 + np.uint64(W1)) & mask
        p0 = m0 * c0            # exact: both factors < 2^32, product < 2^64
        p1 = m1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0), lo1, (hi0 ^ c3 ^ k1), lo0
    return c0, c1, c2, c3


def seed_key(seed):
    """Split a 64-bit seed into the two key words (low word first)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return seed & MASK32, seed >> 32


def uniform_open01(x):
    """Map a 32-bit word to (x + 1/2) / 2^32, a uniform draw in (0, 1), fp64."""
    return (np.asarray(x, dtype=np.float64) + 0.5) * 2.0 ** -32


def box_muller(x0, x1):
    """Standard normal from two words: sqrt(-2 ln u0) * cos(2 pi u1), fp64."""
    u0 = uniform_open01(x0)
    u1 = uniform_open01(x1)
    return np.sqrt(-2.0 * np.log(u0)) * np.cos(2.0 * np.pi * u1)


def box_muller_pair16(x):
    """Two independent standard normals from the two 16-bit halves of a word (fp64).

    The radius draw is u = ((x & 0xFFFF) + 1/2) / 2^16, in (0, 1), from the low
    half. The angle draw is v = (x >> 16) / 2^16, in [0, 1), from the high half.
    The pair is sqrt(-2 ln u) times (cos 2 pi v, sin 2 pi v): the two outputs of
    Box and Muller, "A Note on the Generation of Random Normal Deviates" (1958),
    which are independent N(0, 1). The radius is at most sqrt(-2 ln 2^-17) = 4.85.
    """
    x = np.asarray(x, dtype=np.uint64)
    u = (x & np.uint64(0xFFFF)).astype(np.float64) * 2.0 ** -16 + 2.0 ** -17
    v = (x >> np.uint64(16)).astype(np.float64) * 2.0 ** -16
    r = np.sqrt(-2.0 * np.log(u))
    return r * np.cos(2.0 * np.pi * v), r * np.sin(2.0 * np.pi * v)


def gaussian(seed, c0, c1, c2, stream):
    """fp64 standard normals at counters (c0, c1, c2, stream) under ``seed``."""
    k0, k1 = seed_key(seed)
    x0, x1, _, _ = philox4x32_10(c0, c1, c2, stream, k0, k1)
    return box_muller(x0, x1)
