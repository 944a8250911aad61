"""Parity of the paged decode, causal prefill and KIVI-key workloads at full size.

Each test builds its workload as bench.py does and launches the kernels at
that size. The oracle cannot process the whole workload, so a few sampled
groups are checked. Their inputs (sketch bits and norms, value codes, scales
and zeros, projected queries) are overwritten with the oracle's before the
timed-path launch. So no expected value comes from the CUDA path, and every
other group runs beside them in the same launch. The tolerances are those of
the small-size parity tests.
"""

import math

import numpy as np
import pytest
import torch

import bit_kv_cache_qjl_b200 as qjl
import oracle
from bit_kv_cache_qjl_b200 import workloads as wl
from helpers import check_bits, host, oracle_projection
from oracle import kivi

pytestmark = pytest.mark.gpu


def _dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(a).cuda()


def test_prefill_causal_full(cuda_ok):
    """32 heads x 4096 tokens, dense m = 256 with bf16 S: sketch, 2-bit values, the projection of
    every position (the tensor-core projection) and the causal prefill, sampled query rows."""
    G, L, d, m = 32, 4096, 128, 256
    P = qjl.Projection(2, d, m, "dense", s_bf16=True)
    O = oracle_projection(P)
    keys, vals = wl.decode_kv("cuda", B=1, H=G, N=L, d=d)
    keys, vals = keys.reshape(-1, d), vals.reshape(-1, d)
    q = wl.normal((G * L, d), 407, "cuda")
    bits, norms = qjl.quantize_keys(P, keys)
    codes, sc, zr = qjl.quantize_values_2bit(vals)
    sq = qjl.project_queries(P, q)
    torch.cuda.synchronize()
    # the full-size projection, on sampled rows
    rows = np.sort(np.random.default_rng(11).choice(G * L, size=4096, replace=False))
    qr = host(q[torch.from_numpy(rows).cuda()])
    want_sq = oracle.qjl.project_queries(O, qr)
    tol = 1e-5 * np.linalg.norm(qr, axis=1, keepdims=True) * np.linalg.norm(O.S, axis=1)[None, :]
    assert np.all(np.abs(host(sq[torch.from_numpy(rows).cuda()]) - want_sq) <= tol)
    # sampled heads take the oracle's inputs
    heads = [0, 31]
    ref = {}
    for g in heads:
        sl = slice(g * L, (g + 1) * L)
        ow, onorm, y = oracle.qjl.quantize_keys(O, host(keys[sl]))
        check_bits(host(bits[sl]), ow, y, onorm, m)
        onorm = onorm.astype(np.float32)
        oc, os_, oz = kivi.quantize_values_2bit(host(vals[sl]).astype(np.float32))
        assert np.array_equal(host(codes[sl]), oc)
        osq = oracle.qjl.project_queries(O, host(q[sl])).astype(np.float32)
        bits[sl], norms[sl], sq[sl] = _dev(ow), _dev(onorm), _dev(osq)
        ref[g] = (ow, onorm.astype(np.float64), kivi.dequantize_values(oc, os_, oz, d), osq.astype(np.float64))
    scale = 1.0 / math.sqrt(d)
    out = qjl.prefill_attention(P, bits.view(G, L, -1), norms.view(G, L), codes.view(G, L, -1),
                                sc.view(G, L, -1), zr.view(G, L, -1), sq.view(G, L, m), scale)
    torch.cuda.synchronize()
    qrows = sorted(set([0, 1, 15, 16, 17, 63, 64, 65, 1000, 2047, 2048, 4095] +
                       list(np.random.default_rng(12).choice(L, size=8, replace=False))))
    for g in heads:
        ow, on64, vhat, osq = ref[g]
        got = host(out[g])
        for i in qrows:
            n = i + 1
            est = oracle.qjl.scores(O, ow[None, :n], on64[None, :n], osq[None, i:i + 1])
            want = oracle.attention.decode_attention(est, vhat[None, :n], scale)[0, 0]
            p = oracle.attention.softmax(est[0, 0] * scale)
            bound = 2e-3 * (p @ np.abs(vhat[:n])) + 1e-6
            err = np.abs(got[i] - want)
            assert np.all(err <= bound), (g, i, (err / bound).max())


def test_paged_decode_full(cuda_ok):
    """The D-FQJL decode cache (32 x 32 heads, 16384 tokens) in 256-token pages under a shuffled
    table: one appended key and value per head at the last position, then the paged decode."""
    B, H, N, d, m, T = 32, 32, 16384, 128, 256, 256
    G, pages = B * H, N // T
    P = qjl.Projection(5, d, m, "dfqjl", dither_sigma_rel=0.5)
    O = oracle_projection(P)
    keys, vals = wl.decode_kv("cuda", B=B, H=H, N=N, d=d)
    keys, vals = keys.reshape(-1, d), vals.reshape(-1, d)
    num_pages = G * pages + 64
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(509))[:G * pages]
    table = perm.view(G, pages).to(torch.int32).cuda()
    t = torch.arange(N, device="cuda")
    rows = (table.long()[:, t // T] * T + (t % T)[None, :]).reshape(-1)
    R = num_pages * T
    pool = dict(bits=torch.zeros((R, m // 32), dtype=torch.int32, device="cuda"),
                norms=torch.zeros((R,), dtype=torch.float32, device="cuda"),
                codes=torch.zeros((R, d // 16), dtype=torch.int32, device="cuda"),
                scale=torch.zeros((R, d // 32), dtype=torch.float16, device="cuda"),
                zero=torch.zeros((R, d // 32), dtype=torch.float16, device="cuda"))
    b0, n0 = qjl.quantize_keys(P, keys)
    c0, s0, z0 = qjl.quantize_values_2bit(vals)
    for k, v in (("bits", b0), ("norms", n0), ("codes", c0), ("scale", s0), ("zero", z0)):
        pool[k][rows] = v
    del b0, n0, c0, s0, z0, rows
    table_h = host(table).view(np.int32)
    heads = [0, 777]
    ref = {}
    for g in heads:
        sl = slice(g * N, (g + 1) * N)
        ow, onorm, _ = oracle.qjl.quantize_keys(O, host(keys[sl]), first_token=g * N)
        oc, os_, oz = kivi.quantize_values_2bit(host(vals[sl]).astype(np.float32))
        prow = torch.from_numpy(oracle.paged.group_rows(table_h, T, g, N)).cuda()
        pool["bits"][prow], pool["norms"][prow] = _dev(ow), _dev(onorm.astype(np.float32))
        pool["codes"][prow], pool["scale"][prow], pool["zero"][prow] = _dev(oc), _dev(os_), _dev(oz)
        ref[g] = [ow, onorm.astype(np.float32), oc, os_, oz]
    seq = torch.full((G,), N, dtype=torch.int32, device="cuda")
    cache = qjl.PagedCache(T, table, seq, pool["bits"], pool["norms"], pool["codes"], pool["scale"], pool["zero"])
    pos = torch.full((G,), N - 1, dtype=torch.int32, device="cuda")
    newk = wl.normal((G, d), 511, "cuda", torch.bfloat16)
    newv = wl.normal((G, d), 512, "cuda", torch.bfloat16)
    q = wl.decode_queries("cuda", B=B, H=H, d=d).reshape(-1, d)
    qjl.append_keys(P, cache, newk, pos)
    qjl.append_values_2bit(cache, newv, pos)
    sq = qjl.project_queries(P, q)
    torch.cuda.synchronize()
    # the appends: the dither token of an appended key is its pool row
    for g in heads:
        r = oracle.paged.pool_row(table_h, T, g, N - 1)
        w1, n1, y1 = oracle.qjl.quantize_keys(O, host(newk[g:g + 1]), first_token=r)
        check_bits(host(pool["bits"][r:r + 1]), w1, y1, n1, m)
        np.testing.assert_allclose(host(pool["norms"][r:r + 1]), n1, rtol=1e-5)
        c1, s1, z1 = kivi.quantize_values_2bit(host(newv[g:g + 1]).astype(np.float32))
        assert np.array_equal(host(pool["codes"][r:r + 1]), c1)
        assert np.array_equal(pool["scale"][r:r + 1].cpu().numpy().view(np.uint16), s1.view(np.uint16))
        assert np.array_equal(pool["zero"][r:r + 1].cpu().numpy().view(np.uint16), z1.view(np.uint16))
        # the oracle's appended row goes into the pool and the reference
        pool["bits"][r:r + 1], pool["norms"][r:r + 1] = _dev(w1), _dev(n1.astype(np.float32))
        ow, onorm, oc, os_, oz = ref[g]
        ow[N - 1], onorm[N - 1], oc[N - 1], os_[N - 1], oz[N - 1] = w1[0], n1[0], c1[0], s1[0], z1[0]
    smx = 1.0 / math.sqrt(d)
    out = qjl.decode_attention_paged(P, cache, sq, N, smx)
    torch.cuda.synchronize()
    for g in heads:
        ow, onorm, oc, os_, oz = ref[g]
        osq = oracle.qjl.project_queries(O, host(q[g:g + 1])).reshape(1, 1, m)
        est = oracle.qjl.scores(O, ow[None], onorm.astype(np.float64)[None], osq)
        vhat = kivi.dequantize_values(oc, os_, oz, d)
        want = oracle.attention.decode_attention(est, vhat[None], smx)[0, 0]
        p = oracle.attention.softmax(est[0, 0] * smx)
        bound = 1e-3 * (p @ np.abs(vhat)) + 1e-6
        err = np.abs(host(out[g]) - want)
        assert np.all(err <= bound), (g, (err / bound).max())


def test_kivi_keys_decode_full(cuda_ok):
    """The KIVI per-channel 2-bit key baseline on the decode keys (8 x 32 heads, 32768 keys):
    quantise every key, score one query per head."""
    B, H, N, d = 8, 32, 32768, 128
    G = B * H
    keys = wl.llama_keys("cuda", B=B, H=H, N=N, d=d).reshape(G, N, d)
    q = wl.llama_queries("cuda", B=B, H=H, d=d).reshape(G, 1, d)
    codes, sc, zr = qjl.kivi_quantize_keys_2bit(keys)
    torch.cuda.synchronize()
    heads = [0, 200]
    ref = {}
    for g in heads:
        oc, os_, oz = kivi.quantize_keys_per_channel(keys[g:g + 1].float().cpu().numpy())
        assert np.array_equal(host(codes[g:g + 1]), oc)
        assert np.array_equal(sc[g:g + 1].cpu().numpy().view(np.uint16), os_.view(np.uint16))
        assert np.array_equal(zr[g:g + 1].cpu().numpy().view(np.uint16), oz.view(np.uint16))
        ref[g] = (oc, os_, oz)
    out = qjl.kivi_key_scores(codes, sc, zr, q)
    torch.cuda.synchronize()
    blk = np.arange(N) // 32
    for g in heads:
        oc, os_, oz = ref[g]
        Q = q[g:g + 1].cpu().numpy().astype(np.float64)
        want = kivi.key_scores(oc, os_, oz, Q)
        mag = 3 * np.abs(os_.astype(np.float64))[:, blk, :] + np.abs(oz.astype(np.float64))[:, blk, :]
        tol = 1e-5 * np.einsum("gjc,gnc->gjn", np.abs(Q), mag)
        assert np.all(np.abs(host(out[g:g + 1]) - want) <= tol)
