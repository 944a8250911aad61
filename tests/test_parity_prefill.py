"""Causal prefill attention vs the oracle (GPU).

The GPU is given the oracle's bits, norms, codes, scales and zeros, and Sq, so
only the kernel's arithmetic is compared. Tolerance:
|gpu - oracle| <= 2e-3 * sum_j p_ij |v_hat_j| + 1e-6. P and v_hat enter the
fp16 tensor cores rounded to binary16 (2^-11 relative each); the products
and sums run in fp32, and the 16-bit rounding of Sq moves the scores by
far less. Shapes cover one and several 128-query tiles (a CTA's tile of
queries and of keys), ragged and exact multiples of 128, L = 1, D-FQJL and
P-FQJL, and keys scaled up so that the running max moves by more than 2^8
between key tiles (the output accumulator is then rescaled in TMEM).
"""

import math

import numpy as np
import pytest
import torch

import bit_kv_cache_qjl_b200 as qjl
import oracle
from helpers import host, oracle_projection

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind,G,L,kscale", [("dense", 2, 16, 1.0), ("dense", 3, 100, 1.0), ("dfqjl", 2, 257, 1.0),
                                             ("dense", 1, 1, 1.0), ("pfqjl", 2, 48, 1.0), ("dense", 1, 128, 1.0),
                                             ("dense", 2, 129, 1.0), ("dense", 1, 700, 6.0), ("dfqjl", 2, 384, 4.0),
                                             ("dense", 1, 1000, 1.0)])
def test_prefill(cuda_ok, kind, G, L, kscale):
    d, m = 128, 256
    P = qjl.Projection(41, d, m, kind)
    O = oracle_projection(P)
    rng = np.random.default_rng(3)
    keys = (kscale * rng.standard_normal((G * L, d))).astype(np.float32)
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
