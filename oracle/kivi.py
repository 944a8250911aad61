"""KIVI-style 2-bit per-token value quantisation (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"Vladimir Braverman" page (catalyzex), abstract "KIVI: A Tuning-Free
Asymmetric 2bit Quantization for KV Cache": the value cache is quantised
per token, asymmetrically, to 2 bits. The page gives no group size, rounding
or storage format. Our readings:
  * groups of 32 consecutive channels of one token;
  * zero point z = min of the group, scale s = (max - min) / 3, both stored
    as fp16 (4 levels z, z+s, z+2s, z+3s);
  * code = clamp(round_half_even((v - z) / s), 0, 3), or 0 when s == 0;
  * 16 codes per uint32 word, channel c at bits 2*(c % 16) of word c // 16.

The floating-point steps that decide an integer (the code) are done in fp32,
the precision the kernel uses: s = fp16(fp32((max - min) / 3)), and
t = fp32(fp32(v - z) / s). Dequantisation code * s + z is then exact in fp64.
"""

import numpy as np

GROUP = 32
CODES_PER_WORD = 16


def quantize_values_2bit(V):
    """V [n][d] (fp32-representable) -> (codes [n][d/16] uint32, scale, zero [n][d/32] fp16)."""
    V = np.asarray(V, dtype=np.float32)
    n, d = V.shape
    if d % GROUP:
        raise ValueError("d must be a multiple of 32")
    G = V.reshape(n, d // GROUP, GROUP)
    mn = G.min(axis=2)
    mx = G.max(axis=2)
    zero = mn.astype(np.float16)
    scale = ((mx - mn) / np.float32(3.0)).astype(np.float32).astype(np.float16)
    z32 = zero.astype(np.float32)[:, :, None]
    s32 = scale.astype(np.float32)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = ((G - z32).astype(np.float32) / s32).astype(np.float32)
    code = np.clip(np.rint(t), 0, 3)
    code = np.where(s32 == 0, 0, code).astype(np.uint64).reshape(n, d)
    code = code.reshape(n, d // CODES_PER_WORD, CODES_PER_WORD)
    shifts = np.uint64(2) * np.arange(CODES_PER_WORD, dtype=np.uint64)
    words = (code << shifts).sum(axis=2).astype(np.uint32)
    return words, scale, zero


def unpack_codes(words, d):
    """[n][d/16] uint32 -> [n][d] codes in 0..3."""
    words = np.asarray(words, dtype=np.uint64)
    n = words.shape[0]
    shifts = np.uint64(2) * np.arange(CODES_PER_WORD, dtype=np.uint64)
    return ((words[:, :, None] >> shifts) & np.uint64(3)).reshape(n, d).astype(np.int64)


def dequantize_values(words, scale, zero, d):
    """v_hat = code * s + z, fp64 [n][d]."""
    code = unpack_codes(words, d).reshape(-1, d // GROUP, GROUP).astype(np.float64)
    s = np.asarray(scale, dtype=np.float64)[:, :, None]
    z = np.asarray(zero, dtype=np.float64)[:, :, None]
    return (code * s + z).reshape(-1, d)


# ---------------------------------------------------------------------------
# Keys, per channel (KIVI abstract: the key cache is quantised per channel, the
# value cache per token). Readings, beside those above for the values:
#   * a channel's group is a block of 32 consecutive tokens of one key head (the
#     last block of a ragged N is shorter); zero and scale per (block, channel);
#   * the same level rule: zero = fp16(min), scale = fp16(fp32(max - min) / 3),
#     code = clamp(round_half_even(fp32(fp32(k - zero) / scale)), 0, 3), or 0
#     when scale == 0;
#   * codes are stored per token like the values: channel c of a token at bits
#     2*(c % 16) of word c // 16.
# ---------------------------------------------------------------------------

KEY_BLOCK = 32


def quantize_keys_per_channel(K):
    """K [G][N][d] (fp32-representable) -> (codes [G][N][d/16] uint32, scale, zero [G][ceil(N/32)][d] fp16)."""
    K = np.asarray(K, dtype=np.float32)
    G, N, d = K.shape
    if d % GROUP:
        raise ValueError("d must be a multiple of 32")
    nb = (N + KEY_BLOCK - 1) // KEY_BLOCK
    scale = np.zeros((G, nb, d), dtype=np.float16)
    zero = np.zeros((G, nb, d), dtype=np.float16)
    codes = np.zeros((G, N, d), dtype=np.uint64)
    for b in range(nb):
        blk = K[:, b * KEY_BLOCK:(b + 1) * KEY_BLOCK, :]             # [G][<=32][d]
        mn = blk.min(axis=1)
        mx = blk.max(axis=1)
        z = mn.astype(np.float16)
        s = ((mx - mn) / np.float32(3.0)).astype(np.float32).astype(np.float16)
        z32 = z.astype(np.float32)[:, None, :]
        s32 = s.astype(np.float32)[:, None, :]
        with np.errstate(divide="ignore", invalid="ignore"):
            t = ((blk - z32).astype(np.float32) / s32).astype(np.float32)
        c = np.clip(np.rint(t), 0, 3)
        codes[:, b * KEY_BLOCK:(b + 1) * KEY_BLOCK, :] = np.where(s32 == 0, 0, c).astype(np.uint64)
        scale[:, b], zero[:, b] = s, z
    c = codes.reshape(G, N, d // CODES_PER_WORD, CODES_PER_WORD)
    shifts = np.uint64(2) * np.arange(CODES_PER_WORD, dtype=np.uint64)
    words = (c << shifts).sum(axis=3).astype(np.uint32)
    return words, scale, zero


def dequantize_keys_per_channel(words, scale, zero):
    """k_hat [G][N][d] = code * scale + zero (fp64), the block of token n being n // 32."""
    words = np.asarray(words)
    G, N, w = words.shape
    d = w * CODES_PER_WORD
    code = unpack_codes(words.reshape(G * N, w), d).reshape(G, N, d).astype(np.float64)
    blk = np.arange(N) // KEY_BLOCK
    s = np.asarray(scale, dtype=np.float64)[:, blk, :]
    z = np.asarray(zero, dtype=np.float64)[:, blk, :]
    return code * s + z


def key_scores(words, scale, zero, Q):
    """<q, k_hat> for every (group, query, key): Q [G][J][d] -> [G][J][N] (fp64)."""
    khat = dequantize_keys_per_channel(words, scale, zero)
    return np.einsum("gjc,gnc->gjn", np.asarray(Q, dtype=np.float64), khat)
