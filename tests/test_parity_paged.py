"""Paged cache kernels vs the oracle (GPU).

Appends write one key (sketch) and one value (2-bit codes) per group into page
slots named by a block table. Scores and the fused decode read each group's
first seq_lens[g] tokens through the table. The expected values come from
oracle/paged.py on the same inputs. Tolerances are those of the contiguous
calls (tests/helpers.py): sign bits under the 1e-3 ||k|| margin, norms
relative 1e-5, codes/scale/zero bit-exact, scores 1e-3 c alpha ||k|| ||Sq||_1,
and fused output 1e-3 sum p |v_hat| + 1e-6. Pools start from a sentinel, and
rows that no call should touch must still hold it afterwards.
"""

import math

import numpy as np
import pytest
import torch

import bit_kv_cache_qjl_b200 as qjl
import oracle
from bit_kv_cache_qjl_b200 import workloads as wl
from helpers import check_bits, host, oracle_projection, score_tolerance

pytestmark = pytest.mark.gpu

SENT_BITS = 0x5A5A5A5A


def _layout(G, max_pages, spare, T, seed):
    """A shuffled page assignment: table [G][max_pages] over num_pages = G * max_pages + spare pages."""
    rng = np.random.default_rng(seed)
    num_pages = G * max_pages + spare
    table = rng.permutation(num_pages)[:G * max_pages].reshape(G, max_pages).astype(np.int32)
    return table, num_pages


def _key_pools(num_pages, T, m):
    bits = torch.full((num_pages * T, m // 32), SENT_BITS, dtype=torch.int32, device="cuda")
    norms = torch.full((num_pages * T,), -1.0, dtype=torch.float32, device="cuda")
    return bits, norms


@pytest.mark.parametrize("kind,d,m,dtype,s_bf16", [("dense", 128, 256, torch.bfloat16, True),
                                                   ("dense", 128, 256, torch.float32, False),
                                                   ("dfqjl", 128, 256, torch.bfloat16, True),
                                                   ("pfqjl", 256, 1024, torch.bfloat16, True),
                                                   ("dfqjl", 64, 128, torch.float32, True)])
def test_append_keys(cuda_ok, kind, d, m, dtype, s_bf16):
    G, T, max_pages = 37, 48, 3
    P = qjl.Projection(11, d, m, kind, s_bf16=s_bf16)
    O = oracle_projection(P)
    table, num_pages = _layout(G, max_pages, 5, T, 1)
    rng = np.random.default_rng(2)
    pos = rng.integers(0, max_pages * T, G).astype(np.int32)
    keys = wl.normal((G, d), 12, "cuda", dtype)
    bits, norms = _key_pools(num_pages, T, m)
    cache = qjl.PagedCache(T, torch.from_numpy(table).cuda(), None, bits, norms)
    qjl.append_keys(P, cache, keys, torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    ob = np.full((num_pages * T, m // 32), SENT_BITS, dtype=np.uint32)
    on = np.full(num_pages * T, -1.0)
    pre = oracle.paged.append_keys(O, ob, on, keys.float().cpu().double().numpy(), pos, table, T)
    rows = np.array([oracle.paged.pool_row(table, T, g, int(pos[g])) for g in range(G)])
    gb, gn = host(bits), host(norms)
    check_bits(gb[rows], ob[rows], pre, on[rows], m)
    assert np.allclose(gn[rows], on[rows], rtol=1e-5, atol=0)
    others = np.setdiff1d(np.arange(num_pages * T), rows)
    assert (gb[others] == np.uint32(SENT_BITS)).all() and (gn[others] == -1.0).all()


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 96)])
def test_append_values(cuda_ok, dtype, d):
    G, T, max_pages = 50, 16, 4
    table, num_pages = _layout(G, max_pages, 3, T, 3)
    rng = np.random.default_rng(4)
    pos = rng.integers(0, max_pages * T, G).astype(np.int32)
    v = wl.normal((G, d), 13, "cuda", dtype) * 3
    R = num_pages * T
    codes = torch.full((R, d // 16), SENT_BITS, dtype=torch.int32, device="cuda")
    scale = torch.full((R, d // 32), 7.0, dtype=torch.float16, device="cuda")
    zero = torch.full((R, d // 32), -7.0, dtype=torch.float16, device="cuda")
    cache = qjl.PagedCache(T, torch.from_numpy(table).cuda(), None, None, torch.empty(R, device="cuda"),
                           codes, scale, zero)
    qjl.append_values_2bit(cache, v, torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    oc = np.full((R, d // 16), SENT_BITS, dtype=np.uint32)
    osc = np.full((R, d // 32), 7.0, dtype=np.float16)
    oz = np.full((R, d // 32), -7.0, dtype=np.float16)
    oracle.paged.append_values(oc, osc, oz, v.float().cpu().numpy(), pos, table, T)
    assert np.array_equal(host(codes), oc)
    assert np.array_equal(scale.cpu().numpy().view(np.uint16), osc.view(np.uint16))
    assert np.array_equal(zero.cpu().numpy().view(np.uint16), oz.view(np.uint16))


def _oracle_cache(O, kind_d, G, max_pages, T, spare, seed, values=False):
    """Pools filled by the oracle's own sketch of random keys (and values) under a shuffled table."""
    d, m = O.d, O.m
    table, num_pages = _layout(G, max_pages, spare, T, seed)
    R = num_pages * T
    rng = np.random.default_rng(seed + 100)
    keys = rng.standard_normal((R, d)).astype(np.float32)
    w, n, _ = oracle.qjl.quantize_keys(O, keys)
    pools = {"bits": w, "norms": n.astype(np.float32)}
    if values:
        c, s, z = oracle.kivi.quantize_values_2bit(rng.standard_normal((R, d)).astype(np.float32))
        pools.update(codes=c, scale=s, zero=z)
    return table, num_pages, pools


def _cuda_cache(T, table, seq, pools):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    c = qjl.PagedCache(T, t(table), t(seq.astype(np.int32)), t(pools["bits"].view(np.int32)), t(pools["norms"]))
    if "codes" in pools:
        c.codes, c.scale, c.zero = t(pools["codes"].view(np.int32)), t(pools["scale"]), t(pools["zero"])
    return c


@pytest.mark.parametrize("kind,m,J,T,max_pages", [("dense", 256, 1, 256, 9), ("dense", 256, 2, 48, 50),
                                                  ("dfqjl", 256, 1, 16, 130), ("dense", 512, 1, 1024, 3),
                                                  ("dense", 512, 2, 2048, 2)])
def test_scores_paged(cuda_ok, kind, m, J, T, max_pages):
    G = 9
    P = qjl.Projection(21, 128, m, kind)
    O = oracle_projection(P)
    table, num_pages, pools = _oracle_cache(O, 128, G, max_pages, T, 4, 5)
    L = max_pages * T
    seq = np.array([L, 0, 1, 17, 1023, 1024, 1025, L - 1, 2049], dtype=np.int64)
    seq = np.minimum(seq, L)
    rng = np.random.default_rng(6)
    q = rng.standard_normal((G * J, 128)).astype(np.float32)
    sq = oracle.qjl.project_queries(O, q).astype(np.float32).reshape(G, J, m)
    cache = _cuda_cache(T, table, seq, pools)
    out = torch.full((G, J, L), 12345.0, device="cuda")
    qjl.scores_paged(P, cache, torch.from_numpy(sq).cuda(), L, out=out)
    torch.cuda.synchronize()
    got = host(out)
    want = oracle.paged.scores_paged(O, pools["bits"], pools["norms"].astype(np.float64), table, seq, T,
                                     sq.astype(np.float64), L)
    for g in range(G):
        Lg = int(seq[g])
        rows = oracle.paged.group_rows(table, T, g, Lg)
        if Lg:
            tol = score_tolerance(P.est_scale, pools["norms"][rows][None].astype(np.float64), sq[g:g + 1])[0]
            err = np.abs(got[g, :, :Lg] - want[g, :, :Lg])
            assert np.all(err <= tol), (g, (err / tol).max())
        assert (got[g, :, Lg:] == 12345.0).all()


def test_scores_paged_identity_table_equals_contiguous(cuda_ok):
    G, T, max_pages, m = 6, 256, 8, 256
    P = qjl.Projection(22, 128, m, "dense")
    table = np.arange(G * max_pages, dtype=np.int32).reshape(G, max_pages)
    N = T * max_pages
    keys = wl.normal((G * N, 128), 31, "cuda", torch.bfloat16)
    bits, norms = qjl.quantize_keys(P, keys)
    sq = qjl.project_queries(P, wl.normal((G, 128), 32, "cuda")).view(G, 1, m)
    want = qjl.scores(P, bits.view(G, N, m // 32), norms.view(G, N), sq)
    seq = torch.full((G,), N, dtype=torch.int32, device="cuda")
    cache = qjl.PagedCache(T, torch.from_numpy(table).cuda(), seq, bits, norms)
    got = qjl.scores_paged(P, cache, sq, N)
    torch.cuda.synchronize()
    assert torch.equal(got, want)


@pytest.mark.parametrize("T,max_pages", [(256, 8), (48, 40), (1024, 3)])
def test_decode_attention_paged(cuda_ok, T, max_pages):
    G, d, m = 7, 128, 256
    P = qjl.Projection(23, d, m, "dfqjl")
    O = oracle_projection(P)
    table, num_pages, pools = _oracle_cache(O, d, G, max_pages, T, 2, 7, values=True)
    L = max_pages * T
    seq = np.minimum(np.array([L, 0, 1, 15, 513, L - 3, 1100]), L)
    rng = np.random.default_rng(8)
    sq = oracle.qjl.project_queries(O, rng.standard_normal((G, d)).astype(np.float32)).astype(np.float32)
    cache = _cuda_cache(T, table, seq, pools)
    scale = 1 / math.sqrt(d)
    out = qjl.decode_attention_paged(P, cache, torch.from_numpy(sq).cuda(), L, scale)
    torch.cuda.synchronize()
    got = host(out)
    want, parts = oracle.paged.decode_paged(O, pools["bits"], pools["norms"].astype(np.float64), pools["codes"],
                                            pools["scale"], pools["zero"], table, seq, T, sq.astype(np.float64),
                                            scale, L)
    for g in range(G):
        p, vhat = parts[g]
        tol = 1e-3 * (p[:, None] * np.abs(vhat)).sum(0) + 1e-6 if len(p) else np.full(d, 0.0)
        assert np.all(np.abs(got[g] - want[g]) <= tol), (g, np.abs(got[g] - want[g]).max())
    assert (got[1] == 0).all()                                   # seq_lens 0


def test_decode_paged_identity_table_equals_contiguous(cuda_ok):
    G, T, max_pages, d, m = 5, 512, 4, 128, 256
    P = qjl.Projection(24, d, m, "dfqjl")
    N = T * max_pages
    keys, vals = wl.decode_kv("cuda", B=1, H=G, N=N, d=d)
    bits, norms = qjl.quantize_keys(P, keys.reshape(-1, d))
    codes, sc, zr = qjl.quantize_values_2bit(vals.reshape(-1, d))
    sq = qjl.project_queries(P, wl.normal((G, d), 41, "cuda"))
    want = qjl.decode_attention(P, bits.view(G, N, m // 32), norms.view(G, N), codes.view(G, N, d // 16),
                                sc.view(G, N, d // 32), zr.view(G, N, d // 32), sq.view(G, 1, m), 0.1)
    table = torch.arange(G * max_pages, dtype=torch.int32, device="cuda").view(G, max_pages)
    seq = torch.full((G,), N, dtype=torch.int32, device="cuda")
    cache = qjl.PagedCache(T, table, seq, bits, norms, codes, sc, zr)
    got = qjl.decode_attention_paged(P, cache, sq, N, 0.1)
    torch.cuda.synchronize()
    # the contiguous kernel merges the partial sums of 12 consumer warps and the paged one of 8,
    # so the two add in a different order: equal up to fp32 rounding
    torch.testing.assert_close(got, want.view(G, d), rtol=1e-5, atol=2e-6)


def test_bad_page_entries_are_skipped(cuda_ok):
    # positions and block-table entries out of range: the kernels skip them (no access), the call
    # succeeds, and every well-formed group's result is still right
    G, T, max_pages, d, m = 4, 32, 2, 128, 256
    P = qjl.Projection(25, d, m, "dense")
    table = np.arange(G * max_pages, dtype=np.int32).reshape(G, max_pages)
    table[1, 1] = G * max_pages + 100                            # past num_pages
    table[2, 0] = -5
    num_pages = G * max_pages
    bits, norms = _key_pools(num_pages, T, m)
    cache = qjl.PagedCache(T, torch.from_numpy(table).cuda(), None, bits, norms)
    pos = torch.tensor([3, 40, 2, 10**6], dtype=torch.int32, device="cuda")   # group 3: outside the table
    keys = wl.normal((G, d), 51, "cuda", torch.bfloat16)
    qjl.append_keys(P, cache, keys, pos)
    torch.cuda.synchronize()
    gb = host(bits)
    written = [r for r in range(num_pages * T) if (gb[r] != np.uint32(SENT_BITS)).any()]
    assert written == [oracle.paged.pool_row(table, T, 0, 3)]
    seq = torch.tensor([T * max_pages] * G, dtype=torch.int32, device="cuda")
    cache.seq_lens = seq
    sq = qjl.project_queries(P, wl.normal((G, d), 52, "cuda")).view(G, 1, m)
    out = qjl.scores_paged(P, cache, sq, T * max_pages)
    torch.cuda.synchronize()
    # group 0's scores match the contiguous estimator on its own rows
    rows = torch.arange(T * max_pages, device="cuda")
    want = qjl.scores(P, bits[rows].view(1, -1, m // 32), norms[rows].view(1, -1), sq[:1])
    assert torch.equal(out[:1], want)
