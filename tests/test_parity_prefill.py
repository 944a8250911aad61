"""Causal prefill attention vs the oracle (GPU).

The GPU is given the oracle's bits, norms, codes, scales and zeros, and Sq, so
only the kernel's arithmetic is compared. Tolerance:
|gpu - oracle| <= 2e-3 * sum_j p_ij |v_hat_j| + 1e-6. P and v_hat enter the
fp16 tensor cores rounded to binary16 (2^-11 relative each); the products
and sums run in fp32, and the 23-bit rounding of Sq moves the scores by
far less. Shapes cover one and several 16-query tiles, ragged L, and D-FQJL.
"""

import math

import numpy as np
import pytest
import torch

import bit_kv_cache_qjl_b200 as qjl
import oracle
from helpers import host, oracle_projection

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind,G,L", [("dense", 2, 16), ("dense", 3, 100), ("dfqjl", 2, 257), ("dense", 1, 1),
                                      ("pfqjl", 2, 48)])
def test_prefill(cuda_ok, kind, G, L):
    d, m = 128, 256
    P = qjl.Projection(41, d, m, kind)
    O = oracle_projection(P)
    rng = np.random.default_rng(3)
    keys = rng.standard_normal((G * L, d)).astype(np.float32)
    vals = rng.standard_normal((G * L, d)).astype(np.float32)
    words, norms, _ = oracle.qjl.quantize_keys(O, keys)
    c, s, z = oracle.kivi.quantize_values_2bit(vals)
    q = rng.standard_normal((G * L, d)).astype(np.float32)
    sq = oracle.qjl.project_queries(O, q).astype(np.float32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    scale = 1 / math.sqrt(d)
    out = qjl.prefill_attention(P, t(words.view(np.int32).reshape(G, L, -1)), t(norms.astype(np.float32).reshape(G, L)),
                                t(c.view(np.int32).reshape(G, L, -1)), t(s.reshape(G, L, -1)), t(z.reshape(G, L, -1)),
                                t(sq.reshape(G, L, m)), scale)
    torch.cuda.synchronize()
    n32 = norms.astype(np.float32).astype(np.float64).reshape(G, L)
    est = np.stack([oracle.qjl.scores(O, words.reshape(G, L, -1)[g:g + 1], n32[g:g + 1],
                                      sq.astype(np.float64).reshape(G, L, m)[g:g + 1])[0] for g in range(G)])
    vhat = oracle.kivi.dequantize_values(c, s, z, d).reshape(G, L, d)
    want, p = oracle.attention.prefill_attention(est, vhat, scale)
    tol = 2e-3 * np.einsum("gij,gjd->gid", p, np.abs(vhat)) + 1e-6
    err = np.abs(host(out) - want)
    assert np.all(err <= tol), (err / tol).max()
