"""Pins for the oracle's key sketch, query projection and estimator.

QJL abstract ("Majid Daliri" page): the estimator built from sign(S k),
||k|| and the unquantised S q is unbiased. "Fast Quantized Johnson -
Lindenstrauss Transforms" ("The paper" abstract; "Transcript: The paper's
improvements") says D-FQJL and P-FQJL recover an exactly unbiased estimator.
The pins:
  * Monte-Carlo unbiasedness over 10^4 seeds for dense, D-FQJL and P-FQJL,
    with the mean within 3 standard errors;
  * the closed-form variance ((pi/2)||k||^2||q||^2 - <k,q>^2)/m for dense S;
  * the literal D_g-outside order as a biased negative control;
  * brute-force loops for the projection and for the estimator;
  * closed forms of the FQJL map with D_g = 1;
  * invariants: positive scaling, negation, linearity in q, 1/sqrt(m)
    convergence, and the storage cost of m/8 + 4 bytes per key.
"""

import math

import numpy as np
import pytest

from oracle import hadamard
from oracle import params as P
from oracle import qjl

D_SMALL = 16


def _pair(d, seed=0, corr=0.8):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal(d)
    q = corr * k + math.sqrt(1 - corr * corr) * rng.standard_normal(d)
    return k, q


def _estimates(kind, d, m, seeds, k, q, **kw):
    out = np.empty(len(seeds))
    for t, s in enumerate(seeds):
        proj = P.make_projection(s, d, m, kind, s_bf16=False, **kw)
        words, norms, _ = qjl.quantize_keys(proj, k[None, :])
        sq = qjl.project_queries(proj, q[None, :])
        out[t] = qjl.scores(proj, words[None], norms[None], sq[None])[0, 0, 0]
    return out


@pytest.mark.slow
@pytest.mark.parametrize("kind", [P.KIND_DENSE, P.KIND_DFQJL, P.KIND_PFQJL])
def test_monte_carlo_unbiased(kind):
    k, q = _pair(D_SMALL, seed=kind)
    est = _estimates(kind, D_SMALL, 64, range(10000), k, q)
    se = est.std(ddof=1) / math.sqrt(est.size)
    assert abs(est.mean() - k @ q) < 3 * se, (est.mean(), k @ q, se)


@pytest.mark.slow
def test_literal_dg_outer_order_is_biased():
    """Negative control: D_g outside both Hadamard stages cancels the Gaussian
    diagonal inside sign(.) * (.), so the mean drops to about sqrt(2/pi) <k,q>."""
    k, q = _pair(D_SMALL, seed=7, corr=0.95)
    est = _estimates(P.KIND_PFQJL, D_SMALL, 64, range(4000), k, q, dg_outer=True)
    se = est.std(ddof=1) / math.sqrt(est.size)
    assert abs(est.mean() - k @ q) > 10 * se
    assert 0.7 < est.mean() / (k @ q) < 0.9


@pytest.mark.slow
def test_dense_variance_closed_form():
    d, m = D_SMALL, 64
    k, q = _pair(d, seed=3, corr=0.5)
    est = _estimates(P.KIND_DENSE, d, m, range(10000), k, q)
    want = ((math.pi / 2) * (k @ k) * (q @ q) - (k @ q) ** 2) / m
    dev = est - est.mean()
    var = dev.var(ddof=1)
    se_var = math.sqrt(((dev ** 4).mean() - var ** 2) / est.size)
    assert abs(var - want) < 5 * se_var, (var, want, se_var)


@pytest.mark.slow
def test_error_shrinks_as_one_over_sqrt_m():
    d = D_SMALL
    k, q = _pair(d, seed=5, corr=0.3)
    rms = {}
    for m in (32, 512):
        est = _estimates(P.KIND_DENSE, d, m, range(1500), k, q)
        rms[m] = math.sqrt(((est - k @ q) ** 2).mean())
    ratio = rms[32] / rms[512]
    assert 3.0 < ratio < 5.3, ratio   # sqrt(512/32) = 4


def test_dense_projection_brute_force():
    d, m = 4, 32
    proj = P.make_projection(1, d, m, P.KIND_DENSE)
    rng = np.random.default_rng(1)
    K = rng.standard_normal((3, d))
    Y = qjl.project(proj, K)
    for n in range(3):
        for i in range(m):
            acc = 0.0
            for j in range(d):
                acc += proj.S[i][j] * K[n][j]
            assert abs(Y[n][i] - acc) <= 1e-12 * (1 + abs(acc))


def test_pack_bit_order_brute_force():
    rng = np.random.default_rng(2)
    Y = rng.standard_normal((3, 64))
    Y[0, 5] = 0.0          # sign(0) = +1
    Y[1, 40] = -0.0
    words = qjl.pack_signs(Y)
    for n in range(3):
        for i in range(64):
            bit = (int(words[n][i // 32]) >> (i % 32)) & 1
            assert bit == (1 if Y[n][i] >= 0 else 0)
    assert np.array_equal(qjl.unpack_signs(words, 64), (Y >= 0).astype(np.int64))


def test_estimator_brute_force():
    proj = P.make_projection(4, 8, 32, P.KIND_DFQJL, sigma_rel=0.5)
    rng = np.random.default_rng(4)
    G, J, N, m = 2, 2, 3, 32
    words = rng.integers(0, 2 ** 32, size=(G, N, 1), dtype=np.uint64).astype(np.uint32)
    norms = rng.random((G, N)) + 0.5
    SQ = rng.standard_normal((G, J, m))
    est = qjl.scores(proj, words, norms, SQ)
    c = math.sqrt(math.pi / 2) / m * math.sqrt(1.25)
    for g in range(G):
        for j in range(J):
            for n in range(N):
                acc = 0.0
                for i in range(m):
                    s = 1.0 if (int(words[g][n][0]) >> i) & 1 else -1.0
                    acc += s * SQ[g][j][i]
                assert abs(est[g][j][n] - c * norms[g][n] * acc) < 1e-12 * (1 + abs(acc))


@pytest.mark.parametrize("kind", [P.KIND_DFQJL, P.KIND_PFQJL])
def test_fqjl_map_closed_forms(kind):
    d, m = 16, 32
    proj = P.make_projection(6, d, m, kind)
    X = np.random.default_rng(6).standard_normal((4, d))
    proj.D_g = np.ones_like(proj.D_g)
    Y = qjl.fqjl_map(proj, X)
    for b in range(m // d):
        Yb = Y[:, b * d:(b + 1) * d]
        if kind == P.KIND_DFQJL:
            # sqrt(d) H_n H_n D_r x = sqrt(d) D_r x since H_n is an involution
            assert np.allclose(Yb, math.sqrt(d) * X * proj.D_r[b], atol=1e-12)
        else:
            Hn = hadamard.normalised(d)
            Pm = np.zeros((d, d))
            Pm[np.arange(d), proj.perm[b]] = 1.0
            M = math.sqrt(d) * Hn @ Pm @ Hn @ np.diag(proj.D_r[b])
            assert np.allclose(Yb, X @ M.T, atol=1e-12)
            assert np.allclose(np.linalg.norm(Yb, axis=1), math.sqrt(d) * np.linalg.norm(X, axis=1))


def test_fqjl_rows_have_unit_gaussian_scale():
    """Inner order: given (D_r, Pi), y_i = sum_j H_ij g_j u'_j has variance ||k||^2."""
    d, m = 64, 64
    k, _ = _pair(d, seed=8)
    ys = []
    for s in range(2000):
        proj = P.make_projection(s, d, m, P.KIND_PFQJL)
        ys.append(qjl.project(proj, k[None, :])[0])
    ys = np.concatenate(ys)
    assert abs(ys.var() / (k @ k) - 1.0) < 0.03


def test_invariants():
    d, m = 32, 128
    proj = P.make_projection(9, d, m, P.KIND_DENSE)
    rng = np.random.default_rng(9)
    K = rng.standard_normal((50, d))
    w1, n1, Y = qjl.quantize_keys(proj, K)
    w2, n2, _ = qjl.quantize_keys(proj, 4.0 * K)
    assert np.array_equal(w1, w2) and np.allclose(n2, 4 * n1)
    w3, _, _ = qjl.quantize_keys(proj, -K)
    nz = qjl.unpack_signs(w1, m)[(Y != 0)]
    assert np.array_equal(qjl.unpack_signs(w3, m)[(Y != 0)], 1 - nz)
    q1, q2 = rng.standard_normal((2, d))
    s = lambda q: qjl.scores(proj, w1[None], n1[None], qjl.project_queries(proj, q[None])[None])
    assert np.allclose(s(2 * q1 - 3 * q2), 2 * s(q1) - 3 * s(q2))
    assert qjl.bytes_per_key(256) == 36 and qjl.bytes_per_key(512) == 68


def test_dither_is_applied_before_sign():
    d, m = 16, 32
    proj = P.make_projection(10, d, m, P.KIND_DFQJL, sigma_rel=0.5)
    K = np.random.default_rng(10).standard_normal((5, d))
    _, norms, Y = qjl.quantize_keys(proj, K, first_token=100)
    clean = qjl.fqjl_map(proj, K)
    xi = P.dither(10, d, m, 100 + np.arange(5))
    assert np.allclose(Y, clean + 0.5 * norms[:, None] * xi, atol=1e-12)
    proj0 = P.make_projection(10, d, m, P.KIND_DFQJL, sigma_rel=0.0)
    _, _, Y0 = qjl.quantize_keys(proj0, K)
    assert np.allclose(Y0, clean, atol=1e-12)
