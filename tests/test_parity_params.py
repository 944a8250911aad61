"""Library-drawn projection parameters equal the oracle's independent draw.

Both sides implement Philox4x32-10, Box-Muller and Fisher-Yates from their
published definitions, in separate code (C++ in the library, numpy in the
oracle). Integer draws (D_r signs, permutations) must match exactly. Gaussian
draws must match exactly as fp32 and bf16 values. The only allowed exception
is a last-place difference of fp64 libm between the two hosts' log/cos, and
none is expected.
"""

import numpy as np
import pytest

from bit_kv_cache_qjl_b200 import Projection
from helpers import oracle_projection

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,m,s_bf16", [(128, 256, True), (128, 512, True), (128, 256, False), (96, 64, True)])
def test_dense_matrix_matches_oracle(cuda_ok, d, m, s_bf16):
    P = Projection(7, d, m, "dense", s_bf16=s_bf16)
    O = oracle_projection(P)
    got = P.export("S").numpy().astype(np.float64)
    assert np.array_equal(got, O.S)


@pytest.mark.parametrize("kind,d,m", [("pfqjl", 256, 1024), ("pfqjl", 32, 64), ("dfqjl", 128, 256),
                                      ("pfqjl", 1024, 1024)])
def test_fqjl_parameters_match_oracle(cuda_ok, kind, d, m):
    P = Projection(11, d, m, kind)
    O = oracle_projection(P)
    assert np.array_equal(P.export("D_r").numpy().astype(np.float64), O.D_r)
    assert np.array_equal(P.export("perm").numpy().astype(np.int64), O.perm)
    assert np.array_equal(P.export("D_g").numpy().astype(np.float64), O.D_g)
    est = P.est_scale
    alpha = np.sqrt(1.25) if kind == "dfqjl" else 1.0
    assert abs(est - np.sqrt(np.pi / 2) / m * alpha) < 1e-7 * est
