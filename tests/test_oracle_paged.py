"""Pins of the paged-cache oracle against the contiguous oracle (CPU).

The paged layout is the library's own (the pages name none), so the oracle
defines each paged operation by the contiguous one on the rows the block table
names. These tests pin that reduction: a cache filled one appended token at a
time, under the identity table, equals the contiguous sketch of the same keys
bit for bit (the dither included: pool row = contiguous row). Reads through a
shuffled table equal the contiguous estimator and attention, exactly.
"""

import numpy as np
import pytest

import oracle
from oracle import paged



def _proj(kind, d=32, m=64, seed=3):
    k = {"dense": oracle.params.KIND_DENSE, "dfqjl": oracle.params.KIND_DFQJL, "pfqjl": oracle.params.KIND_PFQJL}[kind]
    return oracle.params.make_projection(seed, d, m, k, s_bf16=True, sigma_rel=0.5, dg_outer=False)


def test_pool_row_brute_force():
    table = np.array([[4, 1], [0, 3]])
    T = 16
    want = {(0, 0): 64, (0, 15): 79, (0, 16): 16, (0, 31): 31, (1, 0): 0, (1, 17): 49}
    for (g, t), r in want.items():
        assert paged.pool_row(table, T, g, t) == r
    assert list(paged.group_rows(table, T, 1, 18)) == list(range(0, 16)) + [48, 49]


@pytest.mark.parametrize("kind", ["dense", "dfqjl", "pfqjl"])
def test_append_one_at_a_time_equals_contiguous(kind):
    P = _proj(kind)
    G, T, pages = 3, 16, 2
    L = T * pages
    rng = np.random.default_rng(7)
    keys = rng.standard_normal((G, L, P.d)).astype(np.float32)
    table = np.arange(G * pages).reshape(G, pages)               # identity: pool row = g * L + t
    bits = np.zeros((G * pages * T, P.m // 32), dtype=np.uint32)
    norms = np.zeros(G * pages * T)
    for t in range(L):
        paged.append_keys(P, bits, norms, keys[:, t], np.full(G, t), table, T)
    w, n, _ = oracle.qjl.quantize_keys(P, keys.reshape(G * L, P.d), first_token=0)
    assert np.array_equal(bits, w)
    assert np.array_equal(norms, n)


def test_append_values_scatter():
    G, T, d = 2, 16, 64
    rng = np.random.default_rng(8)
    v = rng.standard_normal((G, d)).astype(np.float32)
    table = np.array([[3, 0], [1, 2]])
    codes = np.zeros((4 * T, d // 16), dtype=np.uint32)
    scale = np.zeros((4 * T, d // 32), dtype=np.float16)
    zero = np.zeros((4 * T, d // 32), dtype=np.float16)
    pos = np.array([17, 5])
    paged.append_values(codes, scale, zero, v, pos, table, T)
    c, s, z = oracle.kivi.quantize_values_2bit(v)
    rows = [0 * T + 1, 1 * T + 5]                                 # group 0: page table[0][1] = 0, slot 1
    assert np.array_equal(codes[rows], c) and np.array_equal(scale[rows], s) and np.array_equal(zero[rows], z)
    others = np.setdiff1d(np.arange(4 * T), rows)
    assert not codes[others].any() and not scale[others].any()


def _shuffled_cache(P, G, pages, T, rng):
    """Contiguous keys/values [G][pages*T] scattered into a pool under a random page permutation."""
    L = pages * T
    keys = rng.standard_normal((G * L, P.d))
    vals = rng.standard_normal((G * L, P.d)).astype(np.float32)
    w, n, _ = oracle.qjl.quantize_keys(P, keys)
    c, s, z = oracle.kivi.quantize_values_2bit(vals)
    perm = rng.permutation(G * pages)
    table = perm.reshape(G, pages)
    bits = np.zeros_like(w); norms = np.zeros_like(n)
    codes = np.zeros_like(c); scale = np.zeros_like(s); zero = np.zeros_like(z)
    for g in range(G):
        for pi in range(pages):
            src = slice((g * pages + pi) * T, (g * pages + pi + 1) * T)
            dst = slice(table[g, pi] * T, (table[g, pi] + 1) * T)
            bits[dst], norms[dst], codes[dst], scale[dst], zero[dst] = w[src], n[src], c[src], s[src], z[src]
    return (w, n, c, s, z), (bits, norms, codes, scale, zero), table


def test_scores_through_shuffled_table_equal_contiguous():
    P = _proj("dense")
    G, pages, T, J = 3, 3, 16, 2
    rng = np.random.default_rng(9)
    (w, n, _, _, _), (bits, norms, _, _, _), table = _shuffled_cache(P, G, pages, T, rng)
    L = pages * T
    SQ = rng.standard_normal((G, J, P.m))
    seq = np.array([L, 17, 0])
    got = paged.scores_paged(P, bits, norms, table, seq, T, SQ, L)
    want = oracle.qjl.scores(P, w.reshape(G, L, -1), n.reshape(G, L), SQ)
    assert np.array_equal(got[0], want[0])
    # a shorter matrix product may round in another order (BLAS blocking): equal to fp64 rounding
    assert np.allclose(got[1][:, :17], want[1][:, :17], rtol=1e-12, atol=0) and np.isnan(got[1][:, 17:]).all()
    assert np.isnan(got[2]).all()


def test_decode_through_shuffled_table_equals_contiguous():
    P = _proj("dfqjl")
    G, pages, T = 2, 2, 16
    rng = np.random.default_rng(10)
    (w, n, c, s, z), pools, table = _shuffled_cache(P, G, pages, T, rng)
    L = pages * T
    SQ = rng.standard_normal((G, P.m))
    got, _ = paged.decode_paged(P, *pools, table, np.array([L, 0]), T, SQ, 0.25, L)
    est = oracle.qjl.scores(P, w.reshape(G, L, -1), n.reshape(G, L), SQ.reshape(G, 1, -1))
    vhat = oracle.kivi.dequantize_values(c, s, z, P.d).reshape(G, L, P.d)
    want = oracle.attention.decode_attention(est, vhat, 0.25)[:, 0]
    assert np.array_equal(got[0], want[0])
    assert not got[1].any()
