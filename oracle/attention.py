"""Decode attention over sketched keys and 2-bit values (oracle side, fp64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

At one decode step the query attends to every cached token. KIVI abstract
("Vladimir Braverman" page): the whole KV cache is read from GPU memory for
each generated token. The logits are the QJL estimates (QJL abstract,
"Majid Daliri" page) times the softmax scale, and the output is the
softmax-weighted sum of the dequantised values. There is no causal mask: a
single decode query sees the whole context.
"""

import numpy as np


def softmax(x, axis=-1):
    """exp(x - max) / sum exp(x - max) along ``axis`` (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - x.max(axis=axis, keepdims=True))
    return e / e.sum(axis=axis, keepdims=True)


def decode_attention(est, vhat, softmax_scale):
    """est [G][J][N] estimated scores, vhat [G][N][d] -> out [G][J][d] (fp64)."""
    p = softmax(np.asarray(est, dtype=np.float64) * softmax_scale, axis=-1)
    return np.einsum("gjn,gnd->gjd", p, np.asarray(vhat, dtype=np.float64))


def prefill_attention(est, vhat, softmax_scale):
    """Causal prefill: est [G][L][L] (query i, key j) and vhat [G][L][d] -> out [G][L][d] (fp64).

    Query i attends to keys 0..i: the scores of later keys are masked out before
    the softmax. This is the many-query form of decode_attention.
    """
    est = np.asarray(est, dtype=np.float64)
    G, L, _ = est.shape
    mask = np.tril(np.ones((L, L), dtype=bool))
    x = np.where(mask[None], est * softmax_scale, -np.inf)
    p = softmax(x, axis=-1)
    return np.einsum("gij,gjd->gid", p, np.asarray(vhat, dtype=np.float64)), p
