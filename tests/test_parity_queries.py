"""Query projection (unquantised JL map) on the GPU vs the oracle."""

import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_qjl_b200 import Projection, project_queries
from bit_kv_cache_qjl_b200 import workloads as wl
from helpers import host, oracle_projection

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind,d,m,nq,kw", [("dense", 128, 256, 16, dict(s_bf16=False)),
                                             ("dense", 128, 512, 37, dict(s_bf16=True)),
                                             ("pfqjl", 256, 1024, 64, {}),
                                             ("dfqjl", 128, 256, 33, {}),
                                             ("pfqjl", 128, 256, 5, dict(dg_outer=True)),
                                             # many queries (a prefill): the bf16 tensor-core kernel
                                             # with three bf16 parts per query element (bf16 S), the
                                             # warp-per-row kernel (fp32 S)
                                             ("dense", 128, 256, 3000, dict(s_bf16=True)),
                                             ("dense", 128, 512, 1037, dict(s_bf16=True)),
                                             ("dense", 64, 128, 1024, dict(s_bf16=True)),
                                             ("dense", 128, 256, 2000, dict(s_bf16=False))])
def test_project_queries(cuda_ok, kind, d, m, nq, kw):
    P = Projection(21, d, m, kind, **kw)
    q = wl.normal((nq, d), 55, "cuda")
    sq = project_queries(P, q)
    torch.cuda.synchronize()
    O = oracle_projection(P)
    want = oracle.qjl.project_queries(O, host(q))
    qn = np.linalg.norm(host(q), axis=1, keepdims=True)
    if kind == "dense":
        rown = np.linalg.norm(O.S, axis=1)[None, :]
    else:
        rown = np.sqrt(d) * np.abs(O.D_g).max()
    tol = 1e-5 * qn * rown + 1e-30
    err = np.abs(host(sq) - want)
    assert np.all(err <= tol), (err / tol).max()


def test_project_queries_many_strided_and_scaled(cuda_ok):
    """Tensor-core projection of many queries: a row stride above d, and rows whose magnitudes
    span many binades (the three bf16 parts must keep fp32 accuracy at every scale)."""
    d, m, nq, ld = 128, 256, 1500, 136
    P = Projection(23, d, m, "dense", s_bf16=True)
    base = wl.normal((nq, ld), 57, "cuda")
    scale = torch.pow(2.0, torch.linspace(-30, 30, nq, device="cuda"))[:, None]
    qfull = base * scale
    q = qfull[:, :d]
    sq = project_queries(P, q)
    torch.cuda.synchronize()
    O = oracle_projection(P)
    qh = host(q)
    want = oracle.qjl.project_queries(O, qh)
    tol = 1e-5 * np.linalg.norm(qh, axis=1, keepdims=True) * np.linalg.norm(O.S, axis=1)[None, :]
    err = np.abs(host(sq) - want)
    assert np.all(err <= tol), (err / tol).max()
