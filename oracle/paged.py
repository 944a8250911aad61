"""Paged cache: one token appended per group, and reads through a block table (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring).

A decode step adds one token per sequence and then reads the whole cache
(KIVI abstract, "Vladimir Braverman" page). The pages name no cache layout.
The paged layout is the library's own: a pool of pages of T token slots, and
group g's logical token t at pool row block_table[g][t // T] * T + t % T.
The oracle's definitions therefore reduce every paged operation to the
contiguous one. Appending is the key sketch (or the value quantiser) of that
one token, written at its pool row. Reading gathers the group's first
seq_lens[g] pool rows in token order and applies the contiguous estimator or
attention. The D-FQJL dither of an appended key uses its pool row as the token
index, where the contiguous call uses first_token + row.
"""

import numpy as np

from . import attention, kivi, qjl


def pool_row(block_table, page_tokens, g, t):
    """Pool row of group g's logical token t."""
    return int(block_table[g][t // page_tokens]) * page_tokens + t % page_tokens


def group_rows(block_table, page_tokens, g, length):
    """Pool rows of group g's first `length` tokens, in token order."""
    return np.array([pool_row(block_table, page_tokens, g, t) for t in range(length)], dtype=np.int64)


def append_keys(proj, bits_pool, norms_pool, keys, positions, block_table, page_tokens):
    """Sketch keys[g] into the pools at group g's position; returns the pre-sign values [G][m]."""
    keys = np.asarray(keys, dtype=np.float64)
    pre = np.empty((keys.shape[0], proj.m))
    for g in range(keys.shape[0]):
        r = pool_row(block_table, page_tokens, g, int(positions[g]))
        words, norm, y = qjl.quantize_keys(proj, keys[g:g + 1], first_token=r)
        bits_pool[r] = words[0]
        norms_pool[r] = norm[0]
        pre[g] = y[0]
    return pre


def append_values(codes_pool, scale_pool, zero_pool, v, positions, block_table, page_tokens):
    """Quantise v[g] (2-bit, per token) into the pools at group g's position."""
    for g in range(v.shape[0]):
        r = pool_row(block_table, page_tokens, g, int(positions[g]))
        c, s, z = kivi.quantize_values_2bit(np.asarray(v[g:g + 1], dtype=np.float32))
        codes_pool[r], scale_pool[r], zero_pool[r] = c[0], s[0], z[0]


def scores_paged(proj, bits_pool, norms_pool, block_table, seq_lens, page_tokens, SQ, max_len):
    """Estimates [G][J][max_len] over each group's first seq_lens[g] tokens (NaN beyond)."""
    SQ = np.asarray(SQ, dtype=np.float64)
    G, J = SQ.shape[0], SQ.shape[1]
    out = np.full((G, J, max_len), np.nan)
    for g in range(G):
        L = int(min(max(seq_lens[g], 0), max_len))
        if L == 0:
            continue
        rows = group_rows(block_table, page_tokens, g, L)
        out[g, :, :L] = qjl.scores(proj, bits_pool[rows][None], norms_pool[rows][None], SQ[g:g + 1])[0]
    return out


def decode_paged(proj, bits_pool, norms_pool, codes_pool, scale_pool, zero_pool, block_table, seq_lens,
                 page_tokens, SQ, softmax_scale, max_len):
    """Fused decode [G][d] over each group's first seq_lens[g] tokens; a group without tokens gives 0.

    Also returns the softmax weights and dequantised values per group (for tolerances)."""
    SQ = np.asarray(SQ, dtype=np.float64)
    G = SQ.shape[0]
    d = proj.d
    out = np.zeros((G, d))
    parts = []
    for g in range(G):
        L = int(min(max(seq_lens[g], 0), max_len))
        if L == 0:
            parts.append((np.zeros(0), np.zeros((0, d))))
            continue
        rows = group_rows(block_table, page_tokens, g, L)
        est = qjl.scores(proj, bits_pool[rows][None], norms_pool[rows][None], SQ[g:g + 1].reshape(1, 1, -1))
        vhat = kivi.dequantize_values(codes_pool[rows], scale_pool[rows], zero_pool[rows], d)
        out[g] = attention.decode_attention(est, vhat[None], softmax_scale)[0, 0]
        parts.append((attention.softmax(est[0, 0] * softmax_scale), vhat))
    return out, parts
