"""KIVI per-channel 2-bit keys (the baseline of the QJL sketch) vs the oracle (GPU).

Codes, scales and zeros are bit-exact: every step that decides them is an
IEEE round-to-nearest operation on both sides. Scores from the oracle's codes
are within 1e-5 * sum_c |q_c| (3 |scale_c| + |zero_c|), the bound of an fp32
sum of d terms. Shapes cover ragged token blocks, d in {64, 128, 256}, fp32 and
bf16 keys, outlier channels and constant channels.
"""

import numpy as np
import pytest
import torch

import bit_kv_cache_qjl_b200 as qjl
from bit_kv_cache_qjl_b200 import workloads as wl
from helpers import host
from oracle import kivi

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,N,d,dtype", [(3, 100, 128, torch.bfloat16), (2, 64, 64, torch.float32),
                                         (1, 33, 256, torch.bfloat16), (4, 1, 128, torch.float32),
                                         (2, 4096, 128, torch.bfloat16)])
def test_quantize(cuda_ok, G, N, d, dtype):
    k = wl.normal((G, N, d), 61, "cuda") * 2
    k[:, :, 3] *= 10                                                     # an outlier channel
    k[0, :min(N, 32), 7] = 0.5                                           # a constant block
    k = k.to(dtype)
    codes, sc, zr = qjl.kivi_quantize_keys_2bit(k)
    torch.cuda.synchronize()
    oc, os_, oz = kivi.quantize_keys_per_channel(k.float().cpu().numpy())
    assert np.array_equal(host(codes), oc)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), os_.view(np.uint16))
    assert np.array_equal(zr.cpu().numpy().view(np.uint16), oz.view(np.uint16))


@pytest.mark.parametrize("G,N,d,J", [(3, 100, 128, 1), (2, 70, 64, 4), (1, 300, 256, 2), (5, 2048, 128, 1)])
def test_scores(cuda_ok, G, N, d, J):
    rng = np.random.default_rng(7)
    K = (rng.standard_normal((G, N, d)) * 2).astype(np.float32)
    oc, os_, oz = kivi.quantize_keys_per_channel(K)
    Q = rng.standard_normal((G, J, d)).astype(np.float32)
    got = qjl.kivi_key_scores(torch.from_numpy(oc.view(np.int32)).cuda(), torch.from_numpy(os_).cuda(),
                              torch.from_numpy(oz).cuda(), torch.from_numpy(Q).cuda())
    torch.cuda.synchronize()
    want = kivi.key_scores(oc, os_, oz, Q.astype(np.float64))
    blk = np.arange(N) // 32
    mag = 3 * np.abs(os_.astype(np.float64))[:, blk, :] + np.abs(oz.astype(np.float64))[:, blk, :]   # [G][N][d]
    tol = 1e-5 * np.einsum("gjc,gnc->gjn", np.abs(Q.astype(np.float64)), mag)
    assert np.all(np.abs(host(got) - want) <= tol)
