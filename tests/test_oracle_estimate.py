"""Pins for oracle.estimate: the QJL-corrected inner-product estimator.

[JJ] 第六部分 "无偏估计的数学保证": the estimator is unbiased and its variance falls as 1/m.
[JJ] 第二部分 第二步: full-precision query against the 1-bit compressed key.

For s ~ N(0, I): E[sign(<s,r>) <s,q>] = sqrt(2/pi) <q,r>/||r|| and E[<s,q>^2] = ||q||^2, so one
projected row contributes X = nu*gamma*sqrt(pi/2)*sign(<s,r>)*<s,q'> with mean nu*<q',r> and
variance nu^2 (pi/2 gamma^2 ||q||^2 - <q',r>^2).  The tests use these closed forms and the
direct inner product <q, x>; none of them re-calls the oracle's own formula.
"""
import math

import numpy as np
import pytest
from scipy.linalg import hadamard

from oracle import codebook, encode, estimate


def _setup(d, bits, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(d) * rng.lognormal(size=d)
    q = rng.standard_normal(d)
    D = rng.choice([-1.0, 1.0], size=d)
    c, t = codebook.codebook(d, bits)
    return rng, x, q, D, c, t


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_qjl_estimator_unbiased_monte_carlo(bits):
    # 10^5 independent Gaussian rows of S, i.e. 10^5 independent one-row JL draws whose
    # average is the m = 10^5 estimator.
    d, m = 64, 100_000
    rng, x, q, D, c, t = _setup(d, bits, 40 + bits)
    S = rng.standard_normal((m, d))
    enc = encode.encode(x[None], D, S, c, t)
    est = estimate.score_encoded(q[None], enc, D, S, c)[0, 0]
    truth = float(q @ x)
    nu, gamma = enc.norm[0], enc.rnorm[0]
    # q' and r: r is the residual of the rotated unit vector; <q', r> = <q, x>/nu - <q', c[code]>
    H = hadamard(d) / math.sqrt(d)
    qr = H @ (D * q)
    r = enc.y[0] - c[enc.codes[0]]
    var_row = nu ** 2 * (math.pi / 2 * gamma ** 2 * (qr @ qr) - (qr @ r) ** 2)
    se = math.sqrt(var_row / m)
    assert abs(est - truth) < 3 * se, (est, truth, se)


def test_qjl_variance_falls_as_one_over_m():
    d, bits = 64, 2
    rng, x, q, D, c, t = _setup(d, bits, 7)
    ms = [16, 64, 256, 1024]
    variances = []
    for m in ms:
        vals = []
        for _ in range(400):
            S = rng.standard_normal((m, d))
            enc = encode.encode(x[None], D, S, c, t)
            vals.append(estimate.score_encoded(q[None], enc, D, S, c)[0, 0])
        variances.append(np.var(vals))
    slope = np.polyfit(np.log(ms), np.log(variances), 1)[0]
    assert -1.2 < slope < -0.8, slope
    # and the level matches the closed form within sampling error
    enc = encode.encode(x[None], D, rng.standard_normal((1, d)), c, t)
    H = hadamard(d) / math.sqrt(d)
    qr = H @ (D * q)
    r = enc.y[0] - c[enc.codes[0]]
    var_row = enc.norm[0] ** 2 * (math.pi / 2 * enc.rnorm[0] ** 2 * (qr @ qr) - (qr @ r) ** 2)
    for m, v in zip(ms, variances):
        assert v == pytest.approx(var_row / m, rel=0.3)


@pytest.mark.parametrize("d,bits", [(8, 2), (128, 3), (1024, 1)])
def test_mse_only_score_is_inner_product_with_reconstruction(d, bits):
    # With m = 0 the score is exactly <q, x^> with x^ = nu * D H c[code] / sqrt(d).
    rng, x, q, D, c, t = _setup(d, bits, 3)
    X = np.stack([x, 2 * x, -x, rng.standard_normal(d)])
    enc = encode.encode(X, D, np.zeros((0, d)), c, t)
    Q = np.stack([q, rng.standard_normal(d)])
    got = estimate.score_encoded(Q, enc, D, np.zeros((0, d)), c)
    H = hadamard(d) / math.sqrt(d)
    xhat = enc.norm[:, None] * ((c[enc.codes] @ H.T) * D)
    np.testing.assert_allclose(got, Q @ xhat.T, rtol=1e-12, atol=1e-12)


def test_full_estimator_unbiased_over_random_rotations_and_projections():
    # Averaging over independent (D, S) draws: mean estimate -> <q, x>.
    d, bits, m, trials = 32, 2, 32, 4000
    rng = np.random.default_rng(99)
    x = rng.standard_normal(d) * 3
    q = rng.standard_normal(d)
    c, t = codebook.codebook(d, bits)
    vals = []
    for _ in range(trials):
        D = rng.choice([-1.0, 1.0], size=d)
        S = rng.standard_normal((m, d))
        enc = encode.encode(x[None], D, S, c, t)
        vals.append(estimate.score_encoded(q[None], enc, D, S, c)[0, 0])
    vals = np.array(vals)
    assert abs(vals.mean() - q @ x) < 4 * vals.std() / math.sqrt(trials)


def test_zero_norm_key_scores_zero():
    d, m = 16, 32
    rng = np.random.default_rng(1)
    D = rng.choice([-1.0, 1.0], size=d)
    S = rng.standard_normal((m, d))
    c, t = codebook.codebook(d, 2)
    enc = encode.encode(np.zeros((1, d)), D, S, c, t)
    assert estimate.score_encoded(rng.standard_normal((3, d)), enc, D, S, c).tolist() == [[0.0]] * 3


# ---------------------------------------------------------------- structured QJL (SRHT)
@pytest.mark.parametrize("d,m", [(8, 8), (128, 128), (128, 32), (1024, 256)])
def test_srht_matrix_is_signed_hadamard_rows(d, m):
    rng = np.random.default_rng(d + m)
    D2 = rng.choice([-1.0, 1.0], size=d)
    S = encode.srht_matrix(D2, m)
    # scipy's Hadamard matrix (an independent construction), first m rows, columns times D2
    np.testing.assert_array_equal(S, hadamard(d)[:m] * D2[None, :])
    assert set(np.unique(S)) == {-1.0, 1.0}
    np.testing.assert_array_equal(S @ S.T, d * np.eye(m))  # orthogonal rows


def test_srht_estimator_unbiased_monte_carlo():
    """Over 10^5 independent sign vectors D2 the SRHT sign estimator of <q', r> averages to the
    truth within 3 standard errors, at m = d and with m < d rows kept (the transform of D2 * r is
    computed with scipy's Hadamard matrix)."""
    d = 128
    rng = np.random.default_rng(11)
    r = rng.standard_normal(d) * 0.03
    q = rng.standard_normal(d)
    H = hadamard(d).astype(np.float64)
    for m in (128, 32):
        vals = []
        for _ in range(20):
            D2 = rng.choice([-1.0, 1.0], size=(5000, d))
            z = (D2 * r) @ H[:m].T
            p = (D2 * q) @ H[:m].T
            vals.append(math.sqrt(math.pi / 2) / m * np.linalg.norm(r) * np.sum(np.where(z >= 0, 1.0, -1.0) * p, axis=1))
        vals = np.concatenate(vals)
        se = vals.std() / math.sqrt(vals.size)
        assert abs(vals.mean() - r @ q) < 3 * se, (m, vals.mean(), r @ q, se)


def test_srht_oracle_estimator_unbiased_and_variance_falls_with_m():
    """The oracle's encode + estimator with S = srht_matrix(D2, m), averaged over independent D2
    (and rotations D): mean within 4 standard errors of <q, x>; the spread falls as m grows."""
    d, bits, trials = 32, 2, 3000
    rng = np.random.default_rng(5)
    x = rng.standard_normal(d) * 3
    q = rng.standard_normal(d)
    c, t = codebook.codebook(d, bits)
    spread = {}
    for m in (8, 32):
        vals = []
        for _ in range(trials):
            D = rng.choice([-1.0, 1.0], size=d)
            S = encode.srht_matrix(rng.choice([-1.0, 1.0], size=d), m)
            enc = encode.encode(x[None], D, S, c, t)
            vals.append(estimate.score_encoded(q[None], enc, D, S, c)[0, 0])
        vals = np.array(vals)
        assert abs(vals.mean() - q @ x) < 4 * vals.std() / math.sqrt(trials), m
        spread[m] = vals.std()
    assert spread[32] < 0.75 * spread[8]
