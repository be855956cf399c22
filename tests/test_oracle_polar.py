"""Pins for oracle.polar, the PolarQuant first stage ([JJ] 第二部分 第一步: recursive polar transform
of the rotated vector, angles quantized with laws known in advance).

Independent references: adaptive quadrature of the angle laws, Monte-Carlo angles of Gaussian
vectors (a direction uniform on the sphere) against the laws' moments, a d = 8 brute force with
explicit loops over math.atan2 / math.hypot, exact inversion of the unquantized transform, and
the unbiasedness of the QJL-corrected score over independent S.
"""
import math

import numpy as np
import pytest
from scipy import integrate
from scipy.linalg import hadamard

from oracle import polar


@pytest.mark.parametrize("level", [1, 2, 3, 5, 7])
def test_angle_laws_integrate_to_one(level):
    lo, hi = (-math.pi, math.pi) if level == 1 else (0.0, math.pi / 2)
    val, _ = integrate.quad(lambda a: float(polar.angle_density(a, level)), lo, hi, limit=400)
    assert val == pytest.approx(1.0, abs=1e-9)


@pytest.mark.parametrize("level", [2, 3, 4, 7])
def test_angle_laws_match_monte_carlo(level):
    """Angles of Gaussian vectors (uniform directions) at each level: mean and variance against
    the law's quadrature moments, within 4 standard errors."""
    rng = np.random.default_rng(level)
    d = 2 ** 7
    y = rng.standard_normal((40000, d))
    angles, radius = polar.transform(y)
    lv = polar.level_of(d)
    a = angles[:, lv == level].ravel()
    f = lambda t: float(polar.angle_density(t, level))
    m1 = integrate.quad(lambda t: t * f(t), 0, math.pi / 2, limit=400)[0]
    m2 = integrate.quad(lambda t: t * t * f(t), 0, math.pi / 2, limit=400)[0]
    var = m2 - m1 * m1
    # angles of one vector at one level are independent draws; n of them in total
    se = math.sqrt(var / a.size)
    assert abs(a.mean() - m1) < 4 * se, (a.mean(), m1, se)
    assert abs(a.var() - var) < 0.02 * var


def test_level_one_angles_uniform():
    rng = np.random.default_rng(0)
    y = rng.standard_normal((20000, 16))
    a = polar.transform(y)[0][:, :8].ravel()
    hist, _ = np.histogram(a, bins=16, range=(-math.pi, math.pi))
    expect = a.size / 16
    assert np.max(np.abs(hist - expect)) < 5 * math.sqrt(expect)


@pytest.mark.parametrize("level,bits", [(1, 2), (2, 1), (2, 3), (4, 2), (7, 3)])
def test_angle_codebook_lloyd_conditions(level, bits):
    c, t = polar.angle_codebook(level, bits)
    assert np.all(np.diff(c) > 0)
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=1e-12)
    lo, hi = (-math.pi, math.pi) if level == 1 else (0.0, math.pi / 2)
    edges = np.concatenate([[lo], t, [hi]])
    f = lambda a: float(polar.angle_density(a, level))
    for i in range(len(c)):
        mass = integrate.quad(f, edges[i], edges[i + 1], limit=400)[0]
        mom = integrate.quad(lambda a: a * f(a), edges[i], edges[i + 1], limit=400)[0]
        assert mom / mass == pytest.approx(c[i], abs=1e-9)
    # the level laws for k >= 2 are symmetric about pi / 4
    if level >= 2:
        np.testing.assert_allclose(c + c[::-1], math.pi / 2, atol=1e-9)


@pytest.mark.parametrize("d", [2, 8, 128, 1024])
def test_transform_inverts_and_keeps_the_norm(d):
    rng = np.random.default_rng(d)
    y = rng.standard_normal((50, d)) * rng.lognormal(size=d)
    angles, radius = polar.transform(y)
    assert angles.shape == (50, d - 1)
    np.testing.assert_allclose(radius, np.linalg.norm(y, axis=1), rtol=1e-13)
    np.testing.assert_allclose(polar.inverse(angles, radius, d), y, rtol=0, atol=1e-11 * np.max(np.abs(y)))


def test_brute_force_d8():
    """d = 8 with explicit loops: pairs, then pairs of radii, then the last pair."""
    rng = np.random.default_rng(5)
    y = rng.standard_normal((7, 8))
    angles, radius = polar.transform(y)
    for n in range(7):
        v = list(y[n])
        a1 = [math.atan2(v[2 * i + 1], v[2 * i]) for i in range(4)]
        r1 = [math.hypot(v[2 * i], v[2 * i + 1]) for i in range(4)]
        a2 = [math.atan2(r1[2 * i + 1], r1[2 * i]) for i in range(2)]
        r2 = [math.hypot(r1[2 * i], r1[2 * i + 1]) for i in range(2)]
        a3 = [math.atan2(r2[1], r2[0])]
        np.testing.assert_allclose(angles[n], a1 + a2 + a3, rtol=0, atol=1e-15)
        assert radius[n] == pytest.approx(math.hypot(r2[0], r2[1]), rel=1e-15)
        # quantized reconstruction by hand: codes -> centroids -> top-down cos/sin
        codes = polar.quantize_angles(angles[n:n + 1], 8, 2)[0]
        c = [polar.angle_codebook(l, 2)[0] for l in (1, 2, 3)]
        t3 = c[2][codes[6]]
        R2 = [radius[n] * math.cos(t3), radius[n] * math.sin(t3)]
        R1 = []
        for i in range(2):
            t = c[1][codes[4 + i]]
            R1 += [R2[i] * math.cos(t), R2[i] * math.sin(t)]
        yh = []
        for i in range(4):
            t = c[0][codes[i]]
            yh += [R1[i] * math.cos(t), R1[i] * math.sin(t)]
        got = polar.inverse(polar.dequantize_angles(codes[None], 8, 2), radius[n:n + 1], 8)[0]
        np.testing.assert_allclose(got, yh, rtol=0, atol=1e-14)


def test_error_falls_with_bits_and_reconstruction_goes_through_the_rotation():
    d = 128
    rng = np.random.default_rng(9)
    x = rng.standard_normal((200, d)) * rng.lognormal(size=d)
    D = rng.choice([-1.0, 1.0], size=d)
    errs = []
    for b in (1, 2, 3):
        enc = polar.encode(x, D, np.zeros((0, d)), b)
        xh = polar.reconstruct(enc.norm, enc.codes, D, b)
        errs.append(np.mean(np.sum((xh - x) ** 2, axis=1) / np.sum(x ** 2, axis=1)))
        # the stored residual is exactly y / ||x|| - y^ in the rotated domain (scipy's Hadamard)
        H = hadamard(d) / math.sqrt(d)
        y = (x * D) @ H.T
        np.testing.assert_allclose(enc.rnorm, np.linalg.norm(y / enc.norm[:, None] - enc.yhat, axis=1), rtol=1e-10)
    assert all(e2 < e1 for e1, e2 in zip(errs, errs[1:])), errs
    assert errs[-1] < 0.07  # relative squared error at 3 bits per angle


def test_qjl_corrected_score_unbiased_over_projections():
    d, b, m, trials = 32, 2, 32, 3000
    rng = np.random.default_rng(17)
    x = rng.standard_normal(d) * 2
    q = rng.standard_normal(d)
    D = rng.choice([-1.0, 1.0], size=d)
    from oracle import estimate
    vals = []
    for _ in range(trials):
        S = rng.standard_normal((m, d))
        enc = polar.encode(x[None], D, S, b)
        qr, p = estimate.prepare_query(q[None], D, S)
        vals.append(polar.scores(qr, p, enc.norm, enc.codes, enc.rnorm, enc.bits, b)[0, 0])
    vals = np.array(vals)
    assert abs(vals.mean() - q @ x) < 4 * vals.std() / math.sqrt(trials)
    # without the QJL stage the score is exactly <q, x^>
    enc = polar.encode(x[None], D, np.zeros((0, d)), b)
    qr, p = estimate.prepare_query(q[None], D, np.zeros((0, d)))
    xh = polar.reconstruct(enc.norm, enc.codes, D, b)[0]
    assert polar.scores(qr, p, enc.norm, enc.codes, enc.rnorm, enc.bits, b)[0, 0] == pytest.approx(q @ xh, rel=1e-12)


def test_polar_attention_is_softmax_over_reconstructed_keys_and_values():
    """The oracle's decode attention with PolarQuant keys and values (no QJL stage) equals plain
    softmax attention over the vectors rebuilt from the angle codes, computed here directly."""
    from oracle import attention
    d, b, L, hkv, G = 16, 2, 9, 2, 2
    rng = np.random.default_rng(23)
    DK = rng.choice([-1.0, 1.0], size=d)
    DV = rng.choice([-1.0, 1.0], size=d)
    K = rng.standard_normal((b * hkv * L, d))
    V = rng.standard_normal((b * hkv * L, d))
    ek = polar.encode(K, DK, np.zeros((0, d)), b)
    ev = polar.encode(V, DV, np.zeros((0, d)), b)
    kc = attention.Cache(norm=ek.norm, codes=ek.codes)
    vc = attention.Cache(norm=ev.norm, codes=ev.codes)
    q = rng.standard_normal((b, hkv * G, d))
    out = attention.attend_decode(q, kc, vc, [L, L - 4], hkv, DK, np.zeros((0, d)), None, DV, None,
                                  ctx_stride=L, k_polar=b, v_polar=b)
    Kh = polar.reconstruct(ek.norm, ek.codes, DK, b)
    Vh = polar.reconstruct(ev.norm, ev.codes, DV, b)
    for bb in range(b):
        n = [L, L - 4][bb]
        for hq in range(hkv * G):
            h = hq // G
            rows = (bb * hkv + h) * L + np.arange(n)
            lg = Kh[rows] @ q[bb, hq] / math.sqrt(d)
            w = np.exp(lg - lg.max())
            w /= w.sum()
            np.testing.assert_allclose(out[bb, hq], w @ Vh[rows], rtol=1e-12, atol=1e-12)
