"""The arithmetic identities two kernels rely on, checked on the CPU.

* The many-query projection splits an fp32 query element x into three bf16
  parts h = bf16(x), u = bf16(x - h), l = bf16(x - h - u). Both subtractions
  are exact in fp32, |x - h - u - l| <= 2^-27 |x|, and the product of a bf16
  matrix entry with any part is exact in fp32, so three bf16 tensor-core
  products with fp32 accumulation carry the fp32 dot product.
* The prefill dequantises 2-bit codes in half2: the bit pattern 0x6400 | c is
  1024 + c in binary16, and (1024 + c) - 1024 = c exactly.
* The score kernels' shift-window sign sums with four signed base-256 digit
  columns reproduce sum_i b_i Q_i exactly, with no int32 overflow, up to the
  digit grid's bound |Q_i| <= (2^31 - 1) / m.
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


def _window_digits(Q):
    """Per bit i of a 32-bit word: the weight B_i that makes the shift windows exact, as four signed
    base-256 digits. Byte e of (w >> s) is sum_t 2^t b_(8e+s+t); B = K^-1 Q for the unit lower-
    triangular window matrix K, i.e. B_i = sum_k 256^k (Q_(i-8k) - 2 Q_(i-8k-1)) mod 2^32."""
    B = np.zeros(32, dtype=np.int64)
    for i in range(32):
        v = 0
        for k in range(4):
            j = i - 8 * k
            if j < 0:
                break
            v += (int(Q[j]) - (2 * int(Q[j - 1]) if j > 0 else 0)) << (8 * k)
        B[i] = v % (1 << 32)
    dig = np.zeros((32, 4), dtype=np.int64)
    for i in range(32):
        u = int(B[i])
        for c in range(4):
            d = u & 0xFF
            d = d - 256 if d >= 128 else d
            dig[i, c] = d
            u = ((u - d) % (1 << 32)) >> 8
    return dig


def test_shift_window_digits_give_the_exact_sign_sum():
    """The decode-score and prefill kernels' sign sums: eight shifted copies of each sign word as
    u8 operands against four signed digit columns, int32 accumulation, then D0 + 2^8 D1 + 2^16 D2
    + 2^24 D3 in wrapping 32-bit arithmetic. It must equal sum_i b_i Q_i exactly for |Q_i| up to
    (2^31 - 1) / m, and no int32 accumulator may overflow."""
    rng = np.random.default_rng(9)
    for m in (256, 512):
        qmax = (2 ** 31 - 1) // m
        for trial in range(12):
            Q = rng.integers(-qmax, qmax + 1, size=m)
            if trial == 0:
                Q[:] = qmax
            if trial == 1:
                Q[:] = -qmax
            words = rng.integers(0, 1 << 32, size=m // 32, dtype=np.uint64)
            if trial in (0, 1):
                words[:] = (1 << 32) - 1
            D = np.zeros(4, dtype=np.int64)
            for w_idx, w in enumerate(words.tolist()):
                dig = _window_digits(Q[32 * w_idx:32 * (w_idx + 1)])
                for s in range(8):
                    r = w >> s
                    for e in range(4):
                        a = (r >> (8 * e)) & 0xFF
                        D += a * dig[8 * e + s]
                assert np.all(np.abs(D) < 2 ** 31)
            tot = int(sum(int(D[c]) << (8 * c) for c in range(4)) % (1 << 32))
            tot = tot - (1 << 32) if tot >= 1 << 31 else tot
            bits = np.array([(int(words[i // 32]) >> (i % 32)) & 1 for i in range(m)])
            assert tot == int((bits * Q).sum())
            # the estimator's signed sum: 2 tot - sum Q = sum (2 b - 1) Q
            assert 2 * tot - int(Q.sum()) == int(((2 * bits - 1) * Q).sum())


def test_integer_pv_weight_rounding_model():
    """The rounding of a P.V computed as an integer contraction (a design study for the fused decode).

    The weights w_t = p_t * s_t of one 512-token stage are rounded to a (8 nd - 1)-bit
    grid scaled by the stage's max weight, the code sums are exact integers, and the
    zero term is added in float. Over softmaxes from flat to one dominant token, the
    worst error against exact fp64, relative to the fused decode's bound
    1e-3 * sum_t p_t |v_hat_t| + 1e-6, is about 0.5 % (under 1 %) with three int8 digit
    rows and between 1 % and 60 % with two: why three rows were costed.
    """
    rng = np.random.default_rng(0)
    d, N, stage = 128, 16384, 512
    worst = {2: 0.0, 3: 0.0}
    for trial in range(20):
        x = rng.standard_normal(N) * (1.0 + 3.0 * (trial % 4))
        if trial % 5 == 0:
            x[rng.integers(N)] += 30
        p = np.exp(x - x.max())
        codes = rng.integers(0, 4, size=(N, d))
        s = np.abs(rng.standard_normal(N)) * 0.5 + 0.1
        z = rng.standard_normal(N)
        vhat = codes * s[:, None] + z[:, None]
        exact = (p[:, None] * vhat).sum(0)
        bound = 1e-3 * (p[:, None] * np.abs(vhat)).sum(0) + 1e-6
        for nd in (2, 3):
            qmax = (1 << (8 * nd - 1)) - 1
            acc = np.zeros(d)
            for st in range(0, N, stage):
                w = p[st:st + stage] * s[st:st + stage]
                W = w.max()
                wq = np.rint(w / W * qmax)
                acc += (wq[:, None] * codes[st:st + stage]).sum(0) * (W / qmax)
            acc += (p * z).sum()
            worst[nd] = max(worst[nd], (np.abs(acc - exact) / bound).max())
    assert worst[3] < 0.01, worst
    assert 0.01 < worst[2] < 0.6, worst
