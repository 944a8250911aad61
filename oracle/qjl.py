"""QJL key sketch, query projection and asymmetric estimator (oracle side, fp64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

QJL abstract ("Majid Daliri" page, Zandieh, Daliri and Han):
  * a key k is stored as the signs of its JL projection, sign(S k), with no
    quantisation constants. The norm ||k|| is kept beside the bits (the
    estimator needs it);
  * a query q is JL-projected without quantisation (S q);
  * the estimator of <q, k> from (sign(S k), ||k||, S q) is unbiased.
The pages print no formula. For S with iid N(0,1) rows s_i, jointly Gaussian
(s_i.k, s_i.q) give E[sign(s_i.k) (s_i.q)] = sqrt(2/pi) <k,q> / ||k||. So
    est = sqrt(pi/2) / m * ||k|| * sum_i sign(S k)_i (S q)_i
is unbiased, with variance ((pi/2) ||k||^2 ||q||^2 - <k,q>^2) / m.

FQJL ("Fast Quantized Johnson - Lindenstrauss Transforms"): S is replaced by a
composition of randomized Hadamard transforms with a Gaussian second diagonal
("The paper" abstract). P-FQJL puts a random permutation between the two
Hadamard stages ("Key concepts"). D-FQJL adds Gaussian dither before the sign
("Transcript: The paper's improvements"; "Key concepts" says "before applying
the transform", which we read as before the sign quantiser). Our reading of
the order is y = sqrt(d) H_n D_g Pi H_n D_r k, with H_n = H / sqrt(d). This
is "H D" randomized Hadamard transforms composed. It makes every y_i exactly
N(0, ||k||^2) given (D_r, Pi), so the same constant keeps the estimator exactly
unbiased, as the page claims. The literal order D_g H_n Pi H_n D_r (times
sqrt(d)) is available through ``dg_outer``. It is biased, and the tests keep
it as a negative control.

Non-subtractive dither of std sigma_rel * ||k|| before the sign scales the
expectation by 1 / sqrt(1 + sigma_rel^2). The estimator multiplies by
alpha = sqrt(1 + sigma_rel^2) to stay unbiased.

Sign convention: bit = 1 iff the pre-sign value is >= 0 (sign(0) = +1).
Packing: coordinate 32*w + j is bit j of uint32 word w (LSB first).
"""

import numpy as np

from . import hadamard
from . import params as P


def estimator_constant(m):
    """c = sqrt(pi/2) / m."""
    return np.sqrt(np.pi / 2.0) / m


def dither_factor(proj):
    """alpha = sqrt(1 + sigma_rel^2) for D-FQJL, 1 otherwise."""
    return float(np.sqrt(1.0 + proj.sigma_rel ** 2)) if proj.kind == P.KIND_DFQJL else 1.0


def pack_signs(Y):
    """Bits (Y >= 0) packed LSB-first into uint32 words: [n][m] -> [n][m/32]."""
    Y = np.asarray(Y)
    n, m = Y.shape
    bits = (Y >= 0).astype(np.uint64).reshape(n, m // 32, 32)
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    return (bits * weights).sum(axis=2).astype(np.uint32)


def unpack_signs(words, m):
    """Inverse of pack_signs: [n][m/32] uint32 -> [n][m] array of 0/1."""
    words = np.asarray(words, dtype=np.uint64)
    n = words.shape[0]
    shifts = np.arange(32, dtype=np.uint64)
    bits = (words[:, :, None] >> shifts) & np.uint64(1)
    return bits.reshape(n, m).astype(np.int64)


def fqjl_map(proj, X):
    """Unquantised FQJL map of the rows of X: [n][d] -> [n][m] (fp64).

    Block b (output coordinates b*d .. b*d+d-1):
        u  = H_n (D_r^b x)
        u' = Pi^b u          (gather u'[i] = u[pi[i]]; identity for D-FQJL)
        y  = sqrt(d) H_n (D_g^b u')         default order
        y  = sqrt(d) D_g^b (H_n u')         dg_outer (literal order)
    """
    X = np.asarray(X, dtype=np.float64)
    d = proj.d
    Hn = hadamard.normalised(d)
    blocks = []
    for b in range(proj.m // d):
        u = (X * proj.D_r[b]) @ Hn.T
        u = u[:, proj.perm[b]]
        if proj.dg_outer:
            y = np.sqrt(d) * ((u @ Hn.T) * proj.D_g[b])
        else:
            y = np.sqrt(d) * ((u * proj.D_g[b]) @ Hn.T)
        blocks.append(y)
    return np.concatenate(blocks, axis=1)


def project(proj, X):
    """JL map without quantisation: S_eff x (dense) or the FQJL map (fp64)."""
    X = np.asarray(X, dtype=np.float64)
    if proj.kind == P.KIND_DENSE:
        return X @ proj.S.T
    return fqjl_map(proj, X)


def pre_sign(proj, K, first_token=0):
    """The value whose sign is stored: S k, or the FQJL map plus dither (fp64)."""
    K = np.asarray(K, dtype=np.float64)
    Y = project(proj, K)
    if proj.kind == P.KIND_DFQJL and proj.sigma_rel != 0.0:
        norms = np.sqrt((K * K).sum(axis=1))
        tokens = first_token + np.arange(K.shape[0], dtype=np.uint64)
        xi = P.dither(proj.seed, proj.d, proj.m, tokens)
        Y = Y + (proj.sigma_rel * norms)[:, None] * xi
    return Y


def quantize_keys(proj, K, first_token=0):
    """Key sketch: (packed sign words [n][m/32] uint32, norms [n] fp64, pre-sign [n][m])."""
    K = np.asarray(K, dtype=np.float64)
    Y = pre_sign(proj, K, first_token)
    norms = np.sqrt((K * K).sum(axis=1))
    return pack_signs(Y), norms, Y


def project_queries(proj, Q):
    """Sq for each query row: [nq][d] -> [nq][m] (fp64)."""
    return project(proj, Q)


def scores(proj, words, norms, SQ):
    """Estimated <q, k> for every (group, query, key).

    words [G][N][m/32], norms [G][N], SQ [G][J][m] -> est [G][J][N]:
        est = c * alpha * ||k|| * sum_i (2 bit_i - 1) * Sq_i
    """
    words = np.asarray(words)
    G, N, W = words.shape
    m = W * 32
    SQ = np.asarray(SQ, dtype=np.float64).reshape(G, -1, m)
    c = estimator_constant(m) * dither_factor(proj)
    out = np.empty((G, SQ.shape[1], N), dtype=np.float64)
    for g in range(G):
        signs = 2.0 * unpack_signs(words[g], m) - 1.0          # [N][m]
        out[g] = c * (SQ[g] @ signs.T) * np.asarray(norms[g], dtype=np.float64)[None, :]
    return out


def bytes_per_key(m):
    """Storage of one sketched key: m sign bits plus one fp32 norm, no constants."""
    return m // 8 + 4
