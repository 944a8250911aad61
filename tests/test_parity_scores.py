"""Estimator kernels vs the oracle, fed the oracle's bits and norms.

Tolerance: |gpu - oracle| <= 1e-3 * c * alpha * ||k|| * ||Sq||_1 per score.
Covers the mma.sync kernels (one to four queries per group at m = 256, 512),
the tcgen05 kernel (more queries, or m = 1024) and the SIMT kernel for other
m, with 1..64 queries per group, several groups, ragged N and N = 1.
"""

import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_qjl_b200 import Projection, scores
from helpers import host, oracle_projection, score_tolerance

pytestmark = pytest.mark.gpu


def _case(kind, d, m, G, J, N, seed=0):
    P = Projection(31, d, m, kind)
    O = oracle_projection(P)
    rng = np.random.default_rng(seed)
    keys = rng.standard_normal((G * N, d)).astype(np.float32)
    words, norms, _ = oracle.qjl.quantize_keys(O, keys)
    q = rng.standard_normal((G * J, d)).astype(np.float32)
    sq = oracle.qjl.project_queries(O, q).astype(np.float32)        # what the GPU is given
    words = words.reshape(G, N, m // 32)
    norms32 = norms.astype(np.float32).reshape(G, N)
    sq = sq.reshape(G, J, m)
    want = oracle.qjl.scores(O, words, norms32.astype(np.float64), sq.astype(np.float64))
    got = scores(P, torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(norms32).cuda(),
                 torch.from_numpy(sq).cuda())
    torch.cuda.synchronize()
    tol = score_tolerance(P.est_scale, norms32, sq)
    err = np.abs(host(got) - want)
    assert np.all(err <= tol), (err / tol).max()
    return (err / tol).max()


@pytest.mark.parametrize("m,G,J,N", [(256, 3, 1, 1000), (256, 1, 4, 4096), (256, 2, 16, 333), (512, 2, 4, 2049),
                                     (512, 1, 5, 100), (1024, 1, 64, 300), (1024, 2, 1, 1), (256, 4, 3, 17),
                                     (256, 1, 64, 200), (256, 50, 1, 100), (256, 37, 2, 300), (512, 20, 4, 129),
                                     (512, 9, 3, 1000), (256, 300, 1, 7),
                                     # shift-window kernel: whole 1024-key stages, ragged tails, unaligned
                                     # norm rows (N % 4 != 0), N = 1, m = 512 with one and two queries
                                     (256, 2, 1, 3072), (256, 5, 2, 1025), (256, 3, 1, 1), (512, 3, 1, 2500),
                                     (512, 2, 2, 1030), (256, 7, 1, 2051)])
def test_scores_tensor_core(cuda_ok, m, G, J, N):
    _case("dense", 128, m, G, J, N)


# the tcgen05 many-query kernel (more than four queries per group, or m = 1024): every column
# width (8, 16, 32, 64 query slots), ragged tiles, N = 1, and more tiles than CTAs so that a CTA
# spans several groups and rebuilds its tables (two table buffers at m <= 512, one at m = 1024
# with 64 query slots)
@pytest.mark.parametrize("m,G,J,N", [(256, 300, 33, 200), (1024, 200, 64, 130), (512, 7, 12, 1000),
                                     (1024, 3, 5, 4096), (256, 3, 64, 1), (512, 1, 64, 2049),
                                     (1024, 1, 2, 130), (512, 400, 20, 129), (256, 2, 8, 127)])
def test_scores_tcgen05_many(cuda_ok, m, G, J, N):
    _case("dense", 128, m, G, J, N, seed=m + G + J + N)


@pytest.mark.parametrize("m,G,J,N", [(64, 2, 3, 100), (128, 1, 1, 50), (320, 1, 2, 41)])
def test_scores_simt(cuda_ok, m, G, J, N):
    _case("dense", 64, m, G, J, N)


def test_scores_dither_factor(cuda_ok):
    _case("dfqjl", 128, 256, 2, 1, 500)


def test_scores_zero_query(cuda_ok):
    P = Projection(1, 128, 256, "dense")
    bits = torch.randint(-2**31, 2**31 - 1, (1, 64, 8), dtype=torch.int32, device="cuda")
    norms = torch.rand((1, 64), device="cuda")
    sq = torch.zeros((1, 1, 256), device="cuda")
    out = scores(P, bits, norms, sq)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
