"""Shared test helpers: host copies and the tolerance checks the parity tests apply.

Tolerances:
  * bits: bit-exact except where |pre-sign value| < 1e-3 * ||k||. Agreement
    must be >= 99.99 %, and every mismatch must fall inside that margin.
  * scores (from the oracle's bits and norms):
    |gpu - oracle| <= 1e-3 * c * alpha * ||k|| * ||Sq||_1.
  * norms: relative 1e-5 (fp32 accumulation of a d-term sum of squares).
  * projected queries: |gpu - oracle| <= 1e-5 * ||q||_2 * ||S row||_2 per
    coordinate (fp32 accumulation of a d-term dot product), taken as
    1e-5 * ||q|| * sqrt(d) * max|S| for dense S and 1e-5 * ||q|| * max|D_g| * sqrt(d) for FQJL.
  * fused decode output: |gpu - oracle| <= 1e-3 * sum_n p_n |v_hat_n,c| + 1e-6.
"""

import numpy as np
import torch

import oracle


def host(t):
    """CUDA/CPU tensor -> numpy (fp64 for floating types, uint32 view for int32 words)."""
    t = t.detach().cpu()
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    if t.dtype in (torch.bfloat16, torch.float16, torch.float32, torch.float64):
        return t.to(torch.float64).numpy()
    return t.numpy()


def oracle_projection(proj):
    """The oracle's own draw for the same (seed, d, m, kind, options) as a library Projection."""
    return oracle.params.make_projection(proj.seed, proj.d, proj.m, oracle.params.__dict__[
        {"dense": "KIND_DENSE", "dfqjl": "KIND_DFQJL", "pfqjl": "KIND_PFQJL"}[proj.kind]],
        s_bf16=proj.s_bf16, sigma_rel=proj.dither_sigma_rel, dg_outer=proj.dg_outer)


def check_bits(gpu_words, oracle_words, presign, norms, m, margin=1e-3, min_agree=0.9999):
    """Compare packed sign words under the margin rule; returns the agreement fraction."""
    g = oracle.qjl.unpack_signs(np.asarray(gpu_words).reshape(-1, m // 32), m)
    o = oracle.qjl.unpack_signs(np.asarray(oracle_words).reshape(-1, m // 32), m)
    y = np.asarray(presign).reshape(-1, m)
    nrm = np.asarray(norms).reshape(-1, 1)
    bad = g != o
    if bad.any():
        ratio = np.abs(y[bad]) / np.maximum(np.broadcast_to(nrm, y.shape)[bad], 1e-300)
        assert ratio.max() < margin, "bit mismatch outside the margin: |y|/||k|| = %g" % ratio.max()
    agree = 1.0 - bad.mean()
    assert agree >= min_agree, "bit agreement %.6f below %.6f" % (agree, min_agree)
    return agree


def score_tolerance(est_scale, norms, sq):
    """1e-3 * c * alpha * ||k|| * ||Sq||_1, shaped [G, J, N]."""
    l1 = np.abs(np.asarray(sq)).sum(axis=-1)          # [G, J]
    return 1e-3 * est_scale * l1[:, :, None] * np.asarray(norms)[:, None, :]
