"""The arithmetic identities two kernels rely on, checked on the CPU.

* The many-query projection splits an fp32 query element x into three bf16
  parts h = bf16(x), u = bf16(x - h), l = bf16(x - h - u). Both subtractions
  are exact in fp32, |x - h - u - l| <= 2^-27 |x|, and the product of a bf16
  matrix entry with any part is exact in fp32, so three bf16 tensor-core
  products with fp32 accumulation carry the fp32 dot product.
* The prefill dequantises 2-bit codes in half2: the bit pattern 0x6400 | c is
  1024 + c in binary16, and (1024 + c) - 1024 = c exactly.
"""

import numpy as np
import torch


def _bf16(x):
    """Round-to-nearest-even fp32 -> bf16 -> fp32 (torch's CPU conversion)."""
    return x.to(torch.bfloat16).to(torch.float32)


def _values(n, seed):
    g = torch.Generator().manual_seed(seed)
    mant = torch.rand(n, generator=g, dtype=torch.float64) + 1.0
    expo = torch.randint(-60, 61, (n,), generator=g).to(torch.float64)
    sign = torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0).to(torch.float64)
    x = (sign * mant * torch.pow(2.0, expo)).to(torch.float32)
    # bf16 ties and near-ties: 8 significant bits then a trailing 1 (or 1 and more)
    ties = torch.tensor([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -23, 1 - 2.0 ** -24,
                         2.0 ** -126, 3.0e38, -1.5 * 2.0 ** -100], dtype=torch.float32)
    return torch.cat([x, ties, -ties])


def test_three_bf16_parts_are_exact_to_2_pow_minus_27():
    x = _values(1 << 20, 5)
    h = _bf16(x)
    r1 = x - h
    u = _bf16(r1)
    r2 = r1 - u
    lo = _bf16(r2)
    x64, h64, u64, l64 = (t.to(torch.float64) for t in (x, h, u, lo))
    # both fp32 subtractions are exact
    assert torch.equal(r1.to(torch.float64), x64 - h64)
    assert torch.equal(r2.to(torch.float64), x64 - h64 - u64)
    # the three parts carry x to 2^-27 relative
    resid = (x64 - h64 - u64 - l64).abs()
    assert torch.all(resid <= x64.abs() * 2.0 ** -27)


def test_bf16_products_are_exact_in_fp32():
    g = torch.Generator().manual_seed(6)
    s = _bf16(torch.randn(1 << 16, generator=g))
    x = _values(1 << 16, 7)[: 1 << 16]
    for part in (_bf16(x), _bf16(x - _bf16(x))):
        p32 = (s * part).to(torch.float64)
        p64 = s.to(torch.float64) * part.to(torch.float64)
        finite = torch.isfinite(p32) & (p64.abs() >= 2.0 ** -126)     # normal range: no underflow
        assert torch.equal(p32[finite], p64[finite])


def test_half2_code_pattern():
    for c in range(4):
        h = np.array([0x6400 | c], dtype=np.uint16).view(np.float16)[0]
        assert float(h) == 1024 + c
        assert float(np.float16(h - np.float16(1024))) == c
    # the packed extraction: channels i and i + 8 of a 16-code word land in the two halves
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 4, size=16)
    word = int(sum(int(c) << (2 * j) for j, c in enumerate(codes)))
    for i in range(8):
        x = ((word >> (2 * i)) & 0x00030003) | 0x64006400
        lo = np.array([x & 0xFFFF], dtype=np.uint16).view(np.float16)[0]
        hi = np.array([x >> 16], dtype=np.uint16).view(np.float16)[0]
        assert float(lo) - 1024 == codes[i] and float(hi) - 1024 == codes[i + 8]
