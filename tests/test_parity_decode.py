"""Fused decode attention on the GPU vs the oracle.

The inputs are the oracle's bits, norms and 2-bit values, and the same fp32
Sq on both sides. Tolerance per output channel:
|gpu - oracle| <= 1e-3 * sum_n p_n |v_hat_n,c| + 1e-6.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_qjl_b200 import Projection, decode_attention, decode_workspace_bytes
from helpers import host, oracle_projection

pytestmark = pytest.mark.gpu


def _case(kind, d, m, G, J, N, seed=0, scale_keys=1.0):
    P = Projection(41, d, m, kind)
    O = oracle_projection(P)
    rng = np.random.default_rng(seed)
    keys = (scale_keys * rng.standard_normal((G * N, d))).astype(np.float32)
    vals = rng.standard_normal((G * N, d)).astype(np.float32)
    vals = (vals.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    words, norms, _ = oracle.qjl.quantize_keys(O, keys)
    codes, sc, zr = oracle.kivi.quantize_values_2bit(vals)
    q = rng.standard_normal((G * J, d)).astype(np.float32)
    sq = oracle.qjl.project_queries(O, q).astype(np.float32).reshape(G, J, m)
    norms32 = norms.astype(np.float32).reshape(G, N)
    est = oracle.qjl.scores(O, words.reshape(G, N, m // 32), norms32.astype(np.float64), sq.astype(np.float64))
    vhat = oracle.kivi.dequantize_values(codes, sc, zr, d).reshape(G, N, d)
    smx = 1.0 / math.sqrt(d)
    want = oracle.attention.decode_attention(est, vhat, smx)
    p = oracle.attention.softmax(est * smx)
    bound = 1e-3 * np.einsum("gjn,gnd->gjd", p, np.abs(vhat)) + 1e-6
    t = lambda a, dt=None: torch.from_numpy(np.ascontiguousarray(a if dt is None else a.view(dt))).cuda()
    out = decode_attention(P, t(words.reshape(G, N, m // 32), np.int32), t(norms32),
                           t(codes.reshape(G, N, d // 16), np.int32), t(sc.reshape(G, N, d // 32)),
                           t(zr.reshape(G, N, d // 32)), t(sq), smx)
    torch.cuda.synchronize()
    err = np.abs(host(out) - want)
    assert np.all(err <= bound), (err / bound).max()


@pytest.mark.parametrize("kind,d,m,G,J,N", [("dfqjl", 128, 256, 3, 1, 1000), ("dense", 128, 256, 2, 4, 17),
                                            ("dense", 64, 512, 2, 2, 3000), ("pfqjl", 256, 1024, 1, 3, 2500),
                                            ("dense", 32, 256, 4, 1, 1), ("dfqjl", 128, 256, 1, 1, 16384)])
def test_decode_attention(cuda_ok, kind, d, m, G, J, N):
    _case(kind, d, m, G, J, N)


def test_decode_attention_peaked_softmax(cuda_ok):
    """Large keys make the softmax nearly one-hot (stress on max tracking)."""
    _case("dense", 128, 256, 2, 1, 700, seed=3, scale_keys=6.0)


def test_workspace_too_small(cuda_ok):
    import ctypes
    from bit_kv_cache_qjl_b200 import lib
    P = Projection(1, 128, 256, "dense")
    need = decode_workspace_bytes(2, 1, 100, 128)
    z = torch.zeros(1 << 16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(z.data_ptr())
    st = lib().qjl_decode_attention(P.handle, p, p, p, p, p, 2, 100, p, 1, 1.0, p, p, need - 1, None)
    assert st == -5
