"""Pins for the oracle's generator and parameter draws.

The bit stream is pinned by the known-answer vectors published with the
Philox definition (Salmon et al., SC'11, Random123): three (counter, key)
inputs whose ten-round outputs are fixed. These tests also pin what the method relies on: uniform
words and bits, standard-normal Box-Muller output, uniform permutations,
balanced Rademacher signs, independent streams, and the avalanche property
of the block function (one flipped counter bit changes about half of the
output bits). The bf16 rounding is pinned against torch's CPU conversion.
"""

import itertools
import math

import numpy as np
import pytest
import scipy.stats
import torch

from oracle import philox as ph
from oracle import params as P


def _words(n, stream=0, seed=12345):
    k0, k1 = ph.seed_key(seed)
    c = np.arange(n, dtype=np.uint64)
    return ph.philox4x32_10(c, 7, 3, stream, k0, k1)


def test_words_are_uniform():
    x0, x1, x2, x3 = _words(1 << 16)
    for w in (x0, x1, x2, x3):
        hist = np.bincount((w >> np.uint64(24)).astype(np.int64), minlength=256)
        chi2, p = scipy.stats.chisquare(hist)
        assert p > 1e-4, p
        assert int(w.max()) <= 0xFFFFFFFF


def test_every_bit_is_fair():
    words = np.concatenate(_words(1 << 15))
    for b in range(32):
        frac = float(((words >> np.uint64(b)) & np.uint64(1)).mean())
        se = 0.5 / math.sqrt(words.size)
        assert abs(frac - 0.5) < 5 * se, (b, frac)


def test_avalanche_on_counter_and_key():
    k0, k1 = ph.seed_key(99)
    c = np.arange(4096, dtype=np.uint64)
    base = np.stack(ph.philox4x32_10(c, 0, 0, 0, k0, k1))
    for flip in (c ^ np.uint64(1 << 13), c ^ np.uint64(1)):
        other = np.stack(ph.philox4x32_10(flip, 0, 0, 0, k0, k1))
        diff = np.unpackbits((base ^ other).astype(np.uint32).view(np.uint8)).mean()
        assert abs(diff - 0.5) < 0.01
    other = np.stack(ph.philox4x32_10(c, 0, 0, 0, k0 ^ 1, k1))
    diff = np.unpackbits((base ^ other).astype(np.uint32).view(np.uint8)).mean()
    assert abs(diff - 0.5) < 0.01


def test_uniform_open_interval():
    assert ph.uniform_open01(0) == 0.5 * 2.0 ** -32
    assert ph.uniform_open01(0xFFFFFFFF) == 1.0 - 0.5 * 2.0 ** -32
    assert 0.0 < ph.uniform_open01(0) < ph.uniform_open01(0xFFFFFFFF) < 1.0


def test_box_muller_is_standard_normal():
    z = ph.gaussian(2024, np.arange(200000, dtype=np.uint64), 0, 0, ph.STREAM_GAUSS)
    n = z.size
    assert abs(z.mean()) < 5 / math.sqrt(n)
    assert abs(z.var() - 1.0) < 5 * math.sqrt(2.0 / n)
    assert abs((z ** 4).mean() - 3.0) < 5 * math.sqrt(96.0 / n)
    assert scipy.stats.kstest(z, "norm").pvalue > 1e-4


def test_streams_and_blocks_are_uncorrelated():
    c = np.arange(100000, dtype=np.uint64)
    a = ph.gaussian(5, c, 0, 0, ph.STREAM_GAUSS)
    b = ph.gaussian(5, c, 0, 0, ph.STREAM_DITHER)
    e = ph.gaussian(5, c, 0, 1, ph.STREAM_GAUSS)
    for other in (b, e):
        assert abs(np.corrcoef(a, other)[0, 1]) < 5 / math.sqrt(c.size)


def test_dense_matrix_layout_and_stats():
    S = P.dense_gaussian(3, 64, 32)
    assert S.shape == (64, 32)
    # element (i, j) is drawn at index i*d + j
    k0, k1 = ph.seed_key(3)
    x0, x1, _, _ = ph.philox4x32_10(5 * 32 + 7, 0, 0, ph.STREAM_GAUSS, k0, k1)
    assert S[5, 7] == np.float32(ph.box_muller(x0, x1))
    assert np.all(S == S.astype(np.float32))


def test_rademacher_balanced():
    D = P.rademacher(11, 4096, 4)
    assert set(np.unique(D)) == {-1.0, 1.0}
    assert abs(D.mean()) < 5 / math.sqrt(D.size)


def test_fisher_yates_is_uniform_permutation():
    d = 4
    counts = {p: 0 for p in itertools.permutations(range(d))}
    trials = 12000
    for seed in range(trials):
        pi = P.fisher_yates(seed, d, 1)[0]
        counts[tuple(int(v) for v in pi)] += 1
    assert sum(counts.values()) == trials
    chi2, p = scipy.stats.chisquare(list(counts.values()))
    assert p > 1e-4, p


@pytest.mark.parametrize("d", [16, 128, 256])
def test_fisher_yates_is_permutation(d):
    perms = P.fisher_yates(77, d, 4)
    for pi in perms:
        assert sorted(pi.tolist()) == list(range(d))
    assert not np.array_equal(perms[0], perms[1])


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(100000).astype(np.float32)
    # add exact ties: values whose low 16 bits are 0x8000
    u = x.view(np.uint32)
    ties = ((u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    for v in (x, ties):
        want = torch.from_numpy(v.copy()).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.array_equal(P.round_bf16(v), want)


def test_dither_depends_on_absolute_token():
    a = P.dither(9, 16, 32, [10, 11, 12])
    b = P.dither(9, 16, 32, [11, 12])
    assert np.array_equal(a[1:], b)
    big = P.dither(9, 16, 32, [(1 << 32) + 10])
    assert not np.array_equal(big[0], a[0])


def test_dither_is_standard_normal_per_coordinate():
    xi = P.dither(21, 64, 128, np.arange(4000))
    for j in range(8):     # each of the eight coordinates one block yields
        col = xi[:, j::8].ravel()
        assert scipy.stats.kstest(col, "norm").pvalue > 1e-4
    # variance 1 to within the sampling error of 512000 draws
    assert abs(xi.var() - 1.0) < 0.01
    # the fourth moment of N(0, 1) is 3 (the 4.85-sigma cut of the 16-bit radius draw removes
    # a 1.3e-6 tail, far below the sampling error here)
    assert abs((xi ** 4).mean() - 3.0) < 0.05


def test_dither_pairs_are_independent_normals():
    """A Box-Muller pair is two independent N(0,1): its squared radius is
    chi-square with 2 degrees of freedom, and any rotation of the pair is
    again standard normal. Pairs from different words of one block do not
    correlate."""
    xi = P.dither(22, 32, 64, np.arange(5000)).reshape(-1, 8)
    for a in range(0, 8, 2):
        b = a + 1
        r2 = xi[:, a] ** 2 + xi[:, b] ** 2
        assert scipy.stats.kstest(r2, "chi2", args=(2,)).pvalue > 1e-4
        rot = (xi[:, a] + xi[:, b]) / math.sqrt(2.0)
        assert scipy.stats.kstest(rot, "norm").pvalue > 1e-4
    c = np.corrcoef(xi.T)
    assert np.max(np.abs(c - np.eye(8))) < 0.02


def test_dither_prefix_and_block_structure():
    """Coordinates come in eights from one block: the dither of the first m'
    coordinates does not depend on m, and neither on d."""
    a = P.dither(23, 32, 64, [5, 6])
    b = P.dither(23, 64, 256, [5, 6])
    assert np.array_equal(a, b[:, :64])
    assert np.all(np.isfinite(b))
    # the radius draw is never 0 or 1: |xi| is bounded by sqrt(-2 ln 2^-17)
    assert np.max(np.abs(P.dither(24, 128, 1024, np.arange(500)))) < math.sqrt(2 * 17 * math.log(2)) + 1e-9


def test_dither_word_brute_force():
    """Coordinates 8c + 2w and 8c + 2w + 1 of a token, written out from the block's word w:
    u from its low 16 bits, v from its high 16 bits, Box-Muller's cos and sin outputs."""
    seed, t = 0x1234_5678_9ABC_DEF0, (1 << 32) + 77
    xi = P.dither(seed, 32, 64, [t])[0]
    k0, k1 = seed & 0xFFFFFFFF, seed >> 32
    for c in range(8):
        words = ph.philox4x32_10(np.uint64(c), np.uint64(t & 0xFFFFFFFF), np.uint64(t >> 32),
                                 ph.STREAM_DITHER, np.uint64(k0), np.uint64(k1))
        for w in range(4):
            x = int(words[w])
            u = ((x & 0xFFFF) + 0.5) / 65536.0
            v = (x >> 16) / 65536.0
            r = math.sqrt(-2.0 * math.log(u))
            assert abs(xi[8 * c + 2 * w] - r * math.cos(2 * math.pi * v)) < 1e-12
            assert abs(xi[8 * c + 2 * w + 1] - r * math.sin(2 * math.pi * v)) < 1e-12


@pytest.mark.parametrize("ctr,key,want", [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff, 0xffffffff, 0xffffffff, 0xffffffff), (0xffffffff, 0xffffffff),
     (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
])
def test_known_answer_vectors(ctr, key, want):
    """Philox4x32-10 known-answer vectors published with the generator's definition."""
    args = [np.array([v], dtype=np.uint64) for v in ctr + key]
    got = tuple(int(np.asarray(w).ravel()[0]) for w in ph.philox4x32_10(*args))
    assert got == want
