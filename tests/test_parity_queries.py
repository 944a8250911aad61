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
                                             # many queries (a prefill): the warp-per-row kernel
                                             ("dense", 128, 256, 3000, dict(s_bf16=True))])
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
