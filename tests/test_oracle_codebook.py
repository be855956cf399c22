"""Pins for oracle.codebook: the Lloyd-Max codebook of the post-rotation coordinate law.

The law is the density printed in [JJ] 第六部分 "为什么随机旋转这么关键"; Lloyd-Max is named in
[LP] 三.4 and [JJ] 第二部分 第一步.  Independent checks: adaptive quadrature (scipy.integrate.quad)
of the printed density, the closed-form 1-bit centroid, the Gaussian Lloyd-Max quantizer
computed here from scipy.stats.norm (the d -> infinity limit of sqrt(d) X), Monte Carlo over
uniform unit vectors, and the lower bound D_MSE >= 4^-b of [JJ] 第六部分 "量化的理论下界".
"""
import math

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import codebook, encode, rotation

DIMS = [8, 128, 1024]
BITS = [1, 2, 3, 4]


def quad(f, a, b):
    return integrate.quad(f, a, b, limit=400, epsabs=1e-15, epsrel=1e-12)[0]


def printed_density(x, d):
    # f_X(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2), written out again
    # from the page with math.lgamma so that it does not reuse the oracle's constant.
    logc = math.lgamma(d / 2) - math.lgamma((d - 1) / 2) - 0.5 * math.log(math.pi)
    return math.exp(logc) * (1 - x * x) ** ((d - 3) / 2) if abs(x) < 1 else 0.0


@pytest.mark.parametrize("d", DIMS)
def test_density_is_normalised_and_matches_page(d):
    assert quad(lambda x: printed_density(x, d), -1, 1) == pytest.approx(1.0, abs=1e-10)
    xs = np.linspace(-0.9, 0.9, 13) / math.sqrt(d) * 3
    for x in xs:
        assert codebook.density(x, d) == pytest.approx(printed_density(x, d), rel=1e-12)


@pytest.mark.parametrize("d", DIMS)
def test_cdf_matches_quadrature(d):
    for x in np.array([-3.0, -1.0, -0.3, 0.0, 0.5, 2.0]) / math.sqrt(d):
        assert codebook.cdf(x, d) == pytest.approx(quad(lambda s: printed_density(s, d), -1, x), abs=1e-11)


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("bits", BITS)
def test_lloyd_max_fixed_point_conditions(d, bits):
    c, t = codebook.codebook(d, bits)
    L = 1 << bits
    assert c.shape == (L,) and t.shape == (L - 1,)
    assert np.all(np.diff(c) > 0)
    # thresholds are midpoints
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=1e-15)
    # centroids are conditional means, checked by quadrature of the printed density
    edges = np.concatenate(([-1.0], t, [1.0]))
    for i in range(L):
        lo, hi = edges[i], edges[i + 1]
        mass = quad(lambda x: printed_density(x, d), lo, hi)
        mom = quad(lambda x: x * printed_density(x, d), lo, hi)
        assert abs(mom / mass - c[i]) < 1e-9, (i, mom / mass, c[i])


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("bits", BITS)
def test_codebook_is_symmetric(d, bits):
    c, t = codebook.codebook(d, bits)
    np.testing.assert_array_equal(c, -c[::-1])
    assert t[len(t) // 2] == 0.0


@pytest.mark.parametrize("d", DIMS)
def test_one_bit_closed_form(d):
    # E|X| = C_d / (k+1) = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)); the 1-bit cells are X<0, X>=0.
    c, t = codebook.codebook(d, 1)
    expect = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    assert c[1] == pytest.approx(expect, rel=1e-12)
    assert t[0] == pytest.approx(0.0, abs=1e-15)


def gaussian_lloyd_max(bits, iters=20000):
    L = 1 << bits
    c = stats.norm.ppf((np.arange(L) + 0.5) / L)
    for _ in range(iters):
        t = 0.5 * (c[:-1] + c[1:])
        e = np.concatenate(([-np.inf], t, [np.inf]))
        c_new = (stats.norm.pdf(e[:-1]) - stats.norm.pdf(e[1:])) / (stats.norm.cdf(e[1:]) - stats.norm.cdf(e[:-1]))
        if np.max(np.abs(c_new - c)) < 1e-14:
            c = c_new
            break
        c = c_new
    return c


@pytest.mark.parametrize("bits", BITS)
def test_large_d_limit_is_gaussian_lloyd_max(bits):
    # sqrt(d) X -> N(0, 1) as d grows, so sqrt(d) c_d tends to the Gaussian quantizer.
    g = gaussian_lloyd_max(bits)
    errs = []
    for d in (128, 1024, 8192):
        c, _, _ = codebook.lloyd_max(d, bits)
        errs.append(np.max(np.abs(math.sqrt(d) * c - g)))
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 2e-3


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("bits", BITS)
def test_mse_closed_form_matches_quadrature_and_lower_bound(d, bits):
    c, t = codebook.codebook(d, bits)
    mse = codebook.mse_per_coord(d, c, t)
    edges = np.concatenate(([-1.0], t, [1.0]))
    q = sum(quad(lambda x, ci=c[i]: (x - ci) ** 2 * printed_density(x, d), edges[i], edges[i + 1])
            for i in range(len(c)))
    assert mse == pytest.approx(q, rel=1e-8)
    # [JJ] 第六部分 "量化的理论下界": D_MSE >= 1/4^b for a unit vector
    assert d * mse >= 4.0 ** (-bits)


@pytest.mark.parametrize("bits", BITS)
def test_mse_matches_monte_carlo_on_uniform_unit_vectors(bits):
    # For u uniform on the sphere, H D u / sqrt(d) is uniform too, so each rotated coordinate
    # follows f_X exactly and E||u - u^||^2 = d * mse_per_coord.
    d, n = 128, 20000
    rng = np.random.default_rng(11 + bits)
    u = rng.standard_normal((n, d))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    D = rng.choice([-1.0, 1.0], size=d)
    c, t = codebook.codebook(d, bits)
    enc = encode.encode(u, D, np.zeros((0, d)), c, t)
    uhat = rotation.unrotate(c[enc.codes], D)
    err = np.sum((u - uhat) ** 2, axis=1)
    expect = d * codebook.mse_per_coord(d, c, t)
    se = err.std() / math.sqrt(n)
    assert abs(err.mean() - expect) < 4 * se
    assert err.mean() >= 4.0 ** (-bits)


def test_golden_table_is_reproduced():
    # tests/golden/codebooks.json is written by tests/golden/make_golden.py from this oracle;
    # a change to the oracle's arithmetic must regenerate it deliberately.
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "codebooks.json")
    with open(path) as f:
        table = json.load(f)["codebooks"]
    for key, entry in table.items():
        d, b = (int(v) for v in key.split("/"))
        c, t = codebook.codebook(d, b)
        np.testing.assert_allclose(c, [float(v) for v in entry["centroids"]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(t, [float(v) for v in entry["thresholds"]], rtol=0, atol=1e-14)
