"""Lloyd-Max codebook for one coordinate of a randomly rotated unit vector (fp64).

Source.
  [JJ] 第六部分 "为什么随机旋转这么关键": after a random rotation, each coordinate X of a unit
       vector in R^d has the density
           f_X(x) = Gamma(d/2) / (sqrt(pi) * Gamma((d-1)/2)) * (1 - x^2)^((d-3)/2),  x in [-1, 1],
       which does not depend on the data.
  [JJ] 第二部分 第一步 (PolarQuant) and [VC] 第一階段: the quantizer for that known law is the
       optimal scalar (Lloyd-Max) quantizer and needs no per-block normalisation constants.
  [LP] 三.4 "优化理论": Lloyd-Max is the iterative algorithm for the optimal scalar quantizer.

Lloyd's two conditions for 2^b levels c_0 < ... < c_{L-1}:
  thresholds t_i = (c_{i-1} + c_i) / 2                          (nearest-centroid cells)
  centroids  c_i = E[X | t_i <= X < t_{i+1}],  t_0 = -1, t_L = 1  (conditional means)
The iteration alternates them from a quantile start until the centroids stop moving.

Closed forms used (derived from f_X, not from the pages):
  * (1 + X)/2 ~ Beta(a, a) with a = (d-1)/2, so F_X(x) = I_{(1+x)/2}(a, a);
  * int_lo^hi x f_X(x) dx = C_d [(1-lo^2)^(k+1) - (1-hi^2)^(k+1)] / (2(k+1)),  k = (d-3)/2;
  * int_lo^hi x^2 f_X(x) dx = P_d(lo, hi) - (d-1)/d * P_{d+2}(lo, hi), where P_d is the mass
    of the cell under f_X for dimension d (from (1-x^2)^(k+1) = density of dimension d+2).

Pinned by tests/test_oracle_codebook.py: the density integrates to 1 (quadrature), Lloyd's
conditions checked with independent quadrature to 1e-9, the 1-bit closed form
c = +-Gamma(d/2)/(sqrt(pi) Gamma((d+1)/2)), symmetry, the Gaussian Lloyd-Max limit as d grows,
and the MSE lower bound D_MSE >= 4^-b of [JJ] 第六部分 "量化的理论下界".
"""
from __future__ import annotations

import math

import numpy as np
from scipy import special


def density_const(d: int) -> float:
    """C_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))."""
    return math.exp(special.gammaln(d / 2.0) - special.gammaln((d - 1) / 2.0)) / math.sqrt(math.pi)


def density(x, d: int):
    """f_X(x) for a coordinate of a uniformly random unit vector in R^d; 0 outside [-1, 1]."""
    x = np.asarray(x, dtype=np.float64)
    inside = np.abs(x) <= 1.0
    base = np.where(inside, 1.0 - x * x, 0.0)
    return np.where(inside, density_const(d) * base ** ((d - 3) / 2.0), 0.0)


def cdf(x, d: int):
    """F_X(x) = I_{(1+x)/2}((d-1)/2, (d-1)/2)."""
    a = (d - 1) / 2.0
    x = np.clip(np.asarray(x, dtype=np.float64), -1.0, 1.0)
    return special.betainc(a, a, (1.0 + x) / 2.0)


def cell_mass(lo, hi, d: int):
    """P(lo <= X < hi).  Cells in the upper half use F(hi)-F(lo) = F(-lo)-F(-hi) so that the
    small tail masses are differences of small numbers."""
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    upper = lo >= 0.0
    return np.where(upper, cdf(-lo, d) - cdf(-hi, d), cdf(hi, d) - cdf(lo, d))


def cell_first_moment(lo, hi, d: int):
    """int_lo^hi x f_X(x) dx (closed form)."""
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    kp1 = (d - 1) / 2.0
    return density_const(d) * ((1.0 - lo * lo) ** kp1 - (1.0 - hi * hi) ** kp1) / (2.0 * kp1)


def cell_second_moment(lo, hi, d: int):
    """int_lo^hi x^2 f_X(x) dx = P_d(lo, hi) - (d-1)/d * P_{d+2}(lo, hi)."""
    return cell_mass(lo, hi, d) - (d - 1.0) / d * cell_mass(lo, hi, d + 2)


def lloyd_max(d: int, bits: int, tol: float = 1e-13, max_iter: int = 1_000_000):
    """Run Lloyd's iteration for 2**bits levels on f_X.

    Returns (centroids [L], thresholds [L-1], iterations).  Start: the centroids sit at the
    (i + 1/2)/L quantiles of f_X.  Stop: the largest centroid move is below `tol`.
    """
    if d < 3:
        raise ValueError("the density needs d >= 3")
    levels = 1 << bits
    a = (d - 1) / 2.0
    q = (np.arange(levels) + 0.5) / levels
    c = 2.0 * special.betaincinv(a, a, q) - 1.0
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate(([-1.0], t, [1.0]))
        lo, hi = edges[:-1], edges[1:]
        c_new = cell_first_moment(lo, hi, d) / cell_mass(lo, hi, d)
        move = float(np.max(np.abs(c_new - c)))
        c = c_new
        if move < tol:
            break
    # f_X is even, so the Lloyd-Max fixed point is antisymmetric (c_i = -c_{L-1-i}); impose it
    # exactly so that the middle threshold is exactly 0 (ties at y = 0 go to the upper cell).
    c = 0.5 * (c - c[::-1])
    t = 0.5 * (c[:-1] + c[1:])
    return c, t, it


def mse_per_coord(d: int, centroids, thresholds) -> float:
    """E[(X - Q(X))^2] for the quantizer Q with the given cells and reconstruction levels."""
    c = np.asarray(centroids, dtype=np.float64)
    edges = np.concatenate(([-1.0], np.asarray(thresholds, dtype=np.float64), [1.0]))
    lo, hi = edges[:-1], edges[1:]
    m0 = cell_mass(lo, hi, d)
    m1 = cell_first_moment(lo, hi, d)
    m2 = cell_second_moment(lo, hi, d)
    return float(np.sum(m2 - 2.0 * c * m1 + c * c * m0))


_CACHE: dict = {}


def codebook(d: int, bits: int):
    """Cached (centroids, thresholds) for (d, bits)."""
    key = (int(d), int(bits))
    if key not in _CACHE:
        c, t, _ = lloyd_max(d, bits)
        _CACHE[key] = (c, t)
    return _CACHE[key]
