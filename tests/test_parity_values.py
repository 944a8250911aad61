"""2-bit per-token value quantisation on the GPU vs the oracle: bit-exact.

Both sides take the code decision in fp32 with the same IEEE operations, so
codes, scales and zeros must match exactly.
"""

import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_qjl_b200 import quantize_values_2bit
from bit_kv_cache_qjl_b200 import workloads as wl
from helpers import host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,d,dtype", [(1000, 128, torch.bfloat16), (33, 32, torch.bfloat16),
                                       (17, 256, torch.float32), (5, 96, torch.bfloat16), (1, 224, torch.float32)])
def test_values_bit_exact(cuda_ok, n, d, dtype):
    v = wl.normal((n, d), 600 + n, "cuda", dtype)
    codes, scale, zero = quantize_values_2bit(v)
    torch.cuda.synchronize()
    oc, os_, oz = oracle.kivi.quantize_values_2bit(host(v).astype(np.float32))
    assert np.array_equal(host(codes), oc)
    assert np.array_equal(scale.cpu().numpy().view(np.uint16), os_.view(np.uint16))
    assert np.array_equal(zero.cpu().numpy().view(np.uint16), oz.view(np.uint16))


def test_values_constant_groups(cuda_ok):
    v = torch.zeros((3, 64), dtype=torch.bfloat16, device="cuda")
    v[1] = 2.5
    v[2, :32] = -1.0
    codes, scale, zero = quantize_values_2bit(v)
    torch.cuda.synchronize()
    assert torch.all(codes == 0) and torch.all(scale == 0)
    assert torch.equal(zero.float().cpu(), torch.tensor([[0, 0], [2.5, 2.5], [-1.0, 0.0]]))


def test_values_exact_ties(cuda_ok):
    """Values at exact half-levels (t = 0.5, 1.5, 2.5): round-half-even must agree with the
    oracle bit for bit."""
    base = torch.tensor([0.0, 3.0, 0.5, 1.5, 2.5, 1.0, 2.0, 0.75], dtype=torch.float32)
    rows = []
    for scale in (1.0, 0.5, 2.0, 0.25, 3.0, 0.125):
        rows.append((base.repeat(4) * scale + (scale * 7 if scale > 1 else 0.0)))
    v = torch.stack(rows).to(torch.bfloat16).repeat(1, 4).cuda()        # [6, 128]
    codes, scale, zero = quantize_values_2bit(v)
    torch.cuda.synchronize()
    oc, os_, oz = oracle.kivi.quantize_values_2bit(host(v).astype(np.float32))
    assert np.array_equal(host(codes), oc)
    assert np.array_equal(scale.cpu().numpy().view(np.uint16), os_.view(np.uint16))
    # the ties really occur: some codes round half to even
    assert (oracle.kivi.unpack_codes(oc, 128) == 2).any()


def _check(v):
    codes, scale, zero = quantize_values_2bit(v)
    torch.cuda.synchronize()
    oc, os_, oz = oracle.kivi.quantize_values_2bit(host(v).astype(np.float32))
    bad = host(codes) != oc
    assert not bad.any(), "%d of %d code words differ" % (bad.sum(), bad.size)
    assert np.array_equal(scale.cpu().numpy().view(np.uint16), os_.view(np.uint16))
    assert np.array_equal(zero.cpu().numpy().view(np.uint16), oz.view(np.uint16))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_values_quotient_rounding_wide(cuda_ok, dtype):
    """The code decision divides in fp32 with a correctly rounded result. Cover it over
    groups whose magnitudes span 1e-3 .. 1e3 (random full-mantissa fp32, or bf16), both signs,
    offset groups, and many ragged stages: 2^17 tokens x 128 channels against the oracle."""
    n, d = 1 << 17, 128
    g = torch.Generator(device="cpu").manual_seed(77)
    v = torch.randn((n, d), generator=g)
    mag = torch.exp(torch.empty((n, d // 32, 1)).uniform_(-6.9, 6.9, generator=g))
    off = torch.randn((n, d // 32, 1), generator=g) * 3.0
    v = (v.view(n, d // 32, 32) * mag + off * mag).view(n, d)
    _check(v.to(dtype).cuda())


def test_values_constructed_ties(cuda_ok):
    """Groups built so that every channel sits exactly on, or one bf16 step beside, a
    half-level k + 1/2 of its group's step: the cases an approximate quotient gets wrong."""
    g = torch.Generator(device="cpu").manual_seed(78)
    n, d = 4096, 128
    lo = torch.randn((n, d // 32, 1), generator=g)
    step = torch.exp(torch.empty((n, d // 32, 1)).uniform_(-3.0, 3.0, generator=g))
    lvl = torch.randint(0, 7, (n, d // 32, 32), generator=g).float() * 0.5   # 0, 0.5, ..., 3
    lvl[:, :, 0] = 0.0
    lvl[:, :, 1] = 3.0
    v = (lo + lvl * step).to(torch.bfloat16).float()
    # nudge a third of the channels by one bf16 step either way
    bits = v.view(torch.int32)
    nudge = torch.randint(-1, 2, v.shape, generator=g, dtype=torch.int32) << 16
    v = (bits + nudge).view(torch.float32).view(n, d)
    _check(v.to(torch.bfloat16).cuda())
