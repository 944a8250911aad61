"""Projection parameters and dither drawn from a seed (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What is drawn, and which page it comes from:

* Dense QJL: S in R^{m x d} with iid N(0, 1) entries. This is the JL transform
  of the QJL abstract ("Majid Daliri" page). "Fast Quantized Johnson -
  Lindenstrauss Transforms", "The paper", calls it the "dense Gaussian
  projection".
* FQJL: a composition of two randomized Hadamard transforms. The first stage
  uses a Rademacher diagonal D_r. The second uses a Gaussian diagonal D_g
  ("The paper" abstract). P-FQJL adds a uniformly random permutation Pi
  between the two Hadamard stages ("Key concepts"). D-FQJL adds Gaussian
  dither before the sign ("Transcript: The paper's improvements").
  For m > d, m/d independent blocks are stacked, each with its own D_r, Pi
  and D_g.

The pages fix no generator, so this is our reading, and the library follows
the same text. Counters are (c0, c1, c2, c3) = (index_lo, index_hi, block,
stream) under key = seed. Gaussians use Box-Muller on output words 0 and 1 in
fp64 and are then rounded to fp32. Every array below is returned as float64
holding those fp32 (or bf16) values exactly.
"""

from dataclasses import dataclass, field

import numpy as np

from . import philox as ph

KIND_DENSE, KIND_DFQJL, KIND_PFQJL = 0, 1, 2


def round_f32(x):
    """Round fp64 values to fp32 (round to nearest even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x):
    """Round fp32-representable values to bf16 (round to nearest even).

    Keeps the upper 16 bits of the fp32 pattern after adding
    0x7FFF + (bit 16), the textbook round-half-even on the dropped 16 bits.
    """
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def dense_gaussian(seed, m, d):
    """S[i][j] ~ N(0,1) at element index e = i*d + j, stream STREAM_GAUSS, block 0; fp32."""
    e = np.arange(m * d, dtype=np.uint64)
    z = ph.gaussian(seed, e & np.uint64(ph.MASK32), e >> np.uint64(32), 0, ph.STREAM_GAUSS)
    return round_f32(z).reshape(m, d)


def rademacher(seed, d, nblocks):
    """D_r[b][j] = +1 if bit 0 of output word 0 at counter (j, 0, b, 1) is 0, else -1."""
    k0, k1 = ph.seed_key(seed)
    j = np.arange(d, dtype=np.uint64)[None, :]
    b = np.arange(nblocks, dtype=np.uint64)[:, None]
    x0, _, _, _ = ph.philox4x32_10(j, 0, b, ph.STREAM_RADEMACHER, k0, k1)
    return np.where((x0 & np.uint64(1)) == 0, 1.0, -1.0)


def gaussian_diagonal(seed, d, nblocks):
    """D_g[b][j] ~ N(0,1) at counter (j, 0, b, STREAM_GAUSS); fp32."""
    j = np.arange(d, dtype=np.uint64)[None, :]
    b = np.arange(nblocks, dtype=np.uint64)[:, None]
    return round_f32(ph.gaussian(seed, j, 0, b, ph.STREAM_GAUSS))


def fisher_yates(seed, d, nblocks):
    """Uniform permutations of range(d) by Fisher-Yates (Knuth, TAOCP vol. 2, Algorithm P).

    For block b and i = d-1 down to 1, the draw at counter (i, 0, b, STREAM_PERM)
    gives r = w0 * 2^32 + w1, a uniform 64-bit integer. Then
    j = floor(r * (i+1) / 2^64) and pi[i] and pi[j] are swapped. The result is
    used as a gather: (Pi u)[i] = u[pi[i]].
    """
    k0, k1 = ph.seed_key(seed)
    i_all = np.arange(d, dtype=np.uint64)[None, :]
    b_all = np.arange(nblocks, dtype=np.uint64)[:, None]
    x0, x1, _, _ = ph.philox4x32_10(i_all, 0, b_all, ph.STREAM_PERM, k0, k1)
    perms = []
    for b in range(nblocks):
        pi = list(range(d))
        for i in range(d - 1, 0, -1):
            r = (int(x0[b, i]) << 32) | int(x1[b, i])
            j = (r * (i + 1)) >> 64
            pi[i], pi[j] = pi[j], pi[i]
        perms.append(pi)
    return np.array(perms, dtype=np.int64)


def dither(seed, d, m, tokens):
    """D-FQJL dither xi[t][e] ~ N(0,1) for coordinate e = b*d + i of token t.

    The pages ask for Gaussian dither ("Key concepts": non-subtractive Gaussian
    dithering) and fix no generator for it. Here one Philox block gives eight
    coordinates. The block at counter (e // 8, t_lo, t_hi, STREAM_DITHER)
    returns the words x0..x3, and word w gives coordinates 8c + 2w and
    8c + 2w + 1 as the cos and sin outputs of Box-Muller on its two 16-bit
    halves (``philox.box_muller_pair16``).

    ``tokens`` are absolute token indices (first_token + row), so an appended
    key gets the same dither whatever batch it was quantised in.
    """
    tokens = np.asarray(tokens, dtype=np.uint64).reshape(-1, 1)
    c = np.arange(m // 8, dtype=np.uint64).reshape(1, -1)
    k0, k1 = ph.seed_key(seed)
    words = ph.philox4x32_10(c, tokens & np.uint64(ph.MASK32), tokens >> np.uint64(32),
                             ph.STREAM_DITHER, k0, k1)
    outs = []
    for x in words:
        a, b = ph.box_muller_pair16(x)
        outs += [a, b]
    xi = np.stack(outs, axis=-1)                  # [t][c][2w + j], coordinate 8c + 2w + j
    return xi.reshape(tokens.shape[0], m)  # fp64; the library evaluates the same formula in fp32


@dataclass
class Projection:
    """Everything the estimator needs about the random map, as fp64 arrays."""
    kind: int
    d: int
    m: int
    seed: int
    S: np.ndarray = None            # dense: S_eff [m][d]
    D_r: np.ndarray = None          # FQJL: [m/d][d] of +-1
    perm: np.ndarray = None         # FQJL: [m/d][d] gather indices (identity for D-FQJL)
    D_g: np.ndarray = None          # FQJL: [m/d][d]
    sigma_rel: float = 0.0          # D-FQJL dither std relative to ||k||
    dg_outer: bool = False          # literal D_g . H . Pi . H . D_r order (see qjl.fqjl_map)
    extra: dict = field(default_factory=dict)


def make_projection(seed, d, m, kind, s_bf16=True, sigma_rel=0.5, dg_outer=False):
    """Draw the projection for (seed, d, m, kind).

    Dense: S_eff = bf16(S) when ``s_bf16`` (the tensor-core path contracts bf16
    operands, so both keys and queries see the rounded matrix), else fp32 S.
    FQJL: d must be a power of two and m a multiple of d.
    """
    if m % 32 != 0:
        raise ValueError("m must be a multiple of 32")
    if kind == KIND_DENSE:
        S = dense_gaussian(seed, m, d)
        return Projection(kind, d, m, seed, S=round_bf16(S) if s_bf16 else S)
    if d & (d - 1) or m % d:
        raise ValueError("FQJL needs d a power of two and m a multiple of d")
    nb = m // d
    D_r = rademacher(seed, d, nb)
    D_g = gaussian_diagonal(seed, d, nb)
    if kind == KIND_PFQJL:
        perm = fisher_yates(seed, d, nb)
    else:
        perm = np.tile(np.arange(d, dtype=np.int64), (nb, 1))
    return Projection(kind, d, m, seed, D_r=D_r, perm=perm, D_g=D_g,
                      sigma_rel=sigma_rel if kind == KIND_DFQJL else 0.0,
                      dg_outer=dg_outer)
