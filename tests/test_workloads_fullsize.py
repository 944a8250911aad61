"""Parity at the workloads' full sizes, in the launch configuration bench.py times.

The oracle cannot process millions of keys, so each test checks samples it
can compute: whole head slices plus random keys. For the estimator and the
fused decode, the sampled heads' bits, norms and codes are overwritten with
the oracle's before the full-size launch. Their outputs are then compared
with the oracle's, so no expected value comes from the CUDA path.
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


def _sample_rows(n, count, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=count, replace=False))


def _quant_rows_check(P, O, keys_dev, bits, norms, rows):
    idx = torch.from_numpy(rows).cuda()
    K = host(keys_dev[idx])
    # dither (D-FQJL) depends on the absolute token index: check row by row block
    ow = np.empty((len(rows), P.m // 32), dtype=np.uint32)
    onorm = np.empty(len(rows))
    y = np.empty((len(rows), P.m))
    if P.kind == "dfqjl":
        for i, r in enumerate(rows):
            w_, n_, y_ = oracle.qjl.quantize_keys(O, K[i:i + 1], first_token=int(r))
            ow[i], onorm[i], y[i] = w_[0], n_[0], y_[0]
    else:
        ow, onorm, y = oracle.qjl.quantize_keys(O, K)
    check_bits(host(bits[idx]), ow, y, onorm, P.m)
    np.testing.assert_allclose(host(norms[idx]), onorm, rtol=1e-5)


def test_dense_1head_full(cuda_ok):
    w = wl.WORKLOADS["dense_1head"]
    P = qjl.Projection(w["proj_seed"], 128, 256, "dense", s_bf16=False)
    O = oracle_projection(P)
    keys, q = wl.dense_1head("cuda")
    bits, norms = qjl.quantize_keys(P, keys)
    sq = qjl.project_queries(P, q)
    ow, onorm, y = oracle.qjl.quantize_keys(O, host(keys))
    check_bits(host(bits), ow, y, onorm, 256)
    # scores on the oracle's bits (all 4096 x 16)
    ob = torch.from_numpy(ow.view(np.int32).reshape(1, 4096, 8)).cuda()
    on = torch.from_numpy(onorm.astype(np.float32).reshape(1, 4096)).cuda()
    est = qjl.scores(P, ob, on, sq.view(1, 16, 256))
    osq = oracle.qjl.project_queries(O, host(q))
    want = oracle.qjl.scores(O, ow.reshape(1, 4096, 8), onorm.astype(np.float32).astype(np.float64).reshape(1, 4096),
                             osq.reshape(1, 16, 256))
    tol = score_tolerance(P.est_scale, onorm.reshape(1, 4096), osq.reshape(1, 16, 256))
    assert np.all(np.abs(host(est) - want) <= tol)


def _decode_scores_full(P, O, keys, queries, G, N, J, heads):
    """Full-size quantize + project + scores; sampled heads get the oracle's bits."""
    d, m = P.d, P.m
    bits, norms = qjl.quantize_keys(P, keys)
    sq = qjl.project_queries(P, queries)
    rows = _sample_rows(G * N, 1 << 15, 9)
    _quant_rows_check(P, O, keys, bits, norms, rows)
    osq = oracle.qjl.project_queries(O, host(queries)).reshape(G, J, m)
    ow_h, on_h = {}, {}
    for g in heads:
        K = host(keys[g * N:(g + 1) * N])
        ow, onorm, _ = oracle.qjl.quantize_keys(O, K)
        ow_h[g], on_h[g] = ow, onorm.astype(np.float32)
        bits[g * N:(g + 1) * N] = torch.from_numpy(ow.view(np.int32)).cuda()
        norms[g * N:(g + 1) * N] = torch.from_numpy(on_h[g]).cuda()
    est = qjl.scores(P, bits.view(G, N, m // 32), norms.view(G, N), sq.view(G, J, m))
    torch.cuda.synchronize()
    for g in heads:
        want = oracle.qjl.scores(O, ow_h[g][None], on_h[g][None].astype(np.float64), osq[g:g + 1])
        tol = score_tolerance(P.est_scale, on_h[g][None], osq[g:g + 1])
        err = np.abs(host(est[g:g + 1]) - want)
        assert np.all(err <= tol), (g, (err / tol).max())


def test_decode_llama7b_full(cuda_ok):
    B, H, N, d, m = 8, 32, 32768, 128, 256
    P = qjl.Projection(2, d, m, "dense")
    O = oracle_projection(P)
    keys = wl.llama_keys("cuda", B=B, H=H, N=N, d=d).reshape(-1, d)
    q = wl.llama_queries("cuda", B=B, H=H, d=d).reshape(-1, d)
    _decode_scores_full(P, O, keys, q, B * H, N, 1, heads=[0, 77, 160, 255])


def test_gqa_decode_full(cuda_ok):
    B, Hq, Hkv, N, d, m = 16, 32, 8, 131072, 128, 512
    P = qjl.Projection(3, d, m, "dense")
    O = oracle_projection(P)
    keys = wl.gqa_keys("cuda", B=B, Hkv=Hkv, N=N, d=d).reshape(-1, d)
    q = wl.gqa_queries("cuda", B=B, Hq=Hq, d=d).reshape(-1, d)   # head h -> KV head h // 4
    _decode_scores_full(P, O, keys, q, B * Hkv, N, Hq // Hkv, heads=[0, 127])


@pytest.mark.parametrize("m", [256, 1024])
def test_pfqjl_bulk_full(cuda_ok, m):
    n, d = 1 << 24, 256
    P = qjl.Projection(4, d, m, "pfqjl")
    O = oracle_projection(P)
    keys = wl.bulk_keys("cuda", n=n, d=d)
    bits, norms = qjl.quantize_keys(P, keys)
    _quant_rows_check(P, O, keys, bits, norms, _sample_rows(n, 1 << 14, 4))
    # score the first 2^20 keys against 64 queries; the last 4096 of them come from the oracle
    ns = 1 << 20
    q = wl.bulk_queries("cuda", nq=64, d=d)
    sq = qjl.project_queries(P, q)
    tail = np.arange(ns - 4096, ns)
    K = host(keys[ns - 4096:ns])
    ow, onorm, _ = oracle.qjl.quantize_keys(O, K)
    onorm = onorm.astype(np.float32)
    bits[ns - 4096:ns] = torch.from_numpy(ow.view(np.int32)).cuda()
    norms[ns - 4096:ns] = torch.from_numpy(onorm).cuda()
    est = qjl.scores(P, bits[:ns].view(1, ns, m // 32), norms[:ns].view(1, ns), sq.view(1, 64, m))
    torch.cuda.synchronize()
    osq = oracle.qjl.project_queries(O, host(q)).reshape(1, 64, m)
    want = oracle.qjl.scores(O, ow[None], onorm[None].astype(np.float64), osq)
    tol = score_tolerance(P.est_scale, onorm[None], osq)
    err = np.abs(host(est[:, :, ns - 4096:]) - want)
    assert np.all(err <= tol), (err / tol).max()


def test_dfqjl_decode_full(cuda_ok):
    B, H, N, d, m = 32, 32, 16384, 128, 256
    G = B * H
    P = qjl.Projection(5, d, m, "dfqjl", dither_sigma_rel=0.5)
    O = oracle_projection(P)
    keys, vals = wl.decode_kv("cuda", B=B, H=H, N=N, d=d)
    keys, vals = keys.reshape(-1, d), vals.reshape(-1, d)
    q = wl.decode_queries("cuda", B=B, H=H, d=d).reshape(-1, d)
    bits, norms = qjl.quantize_keys(P, keys)              # token index = row (first_token 0)
    codes, sc, zr = qjl.quantize_values_2bit(vals)
    sq = qjl.project_queries(P, q)
    _quant_rows_check(P, O, keys, bits, norms, _sample_rows(G * N, 1 << 11, 5))
    heads = [0, 511, 1023]
    osq = oracle.qjl.project_queries(O, host(q)).reshape(G, 1, m)
    want, bound = {}, {}
    smx = 1.0 / math.sqrt(d)
    for g in heads:
        sl = slice(g * N, (g + 1) * N)
        K = host(keys[sl])
        ow, onorm, _ = oracle.qjl.quantize_keys(O, K, first_token=g * N)
        onorm = onorm.astype(np.float32)
        oc, os_, oz = oracle.kivi.quantize_values_2bit(host(vals[sl]).astype(np.float32))
        assert np.array_equal(host(codes[sl]), oc)
        bits[sl] = torch.from_numpy(ow.view(np.int32)).cuda()
        norms[sl] = torch.from_numpy(onorm).cuda()
        est = oracle.qjl.scores(O, ow[None], onorm[None].astype(np.float64), osq[g:g + 1])
        vhat = oracle.kivi.dequantize_values(oc, os_, oz, d)[None]
        want[g] = oracle.attention.decode_attention(est, vhat, smx)
        p = oracle.attention.softmax(est * smx)
        bound[g] = 1e-3 * np.einsum("gjn,gnd->gjd", p, np.abs(vhat)) + 1e-6
    out = qjl.decode_attention(P, bits.view(G, N, m // 32), norms.view(G, N), codes.view(G, N, d // 16),
                               sc.view(G, N, d // 32), zr.view(G, N, d // 32), sq.view(G, 1, m), smx)
    torch.cuda.synchronize()
    for g in heads:
        err = np.abs(host(out[g:g + 1]) - want[g])
        assert np.all(err <= bound[g]), (g, (err / bound[g]).max())
