"""PolarQuant first stage (fp64): recursive polar transform of the rotated vector and Lloyd-Max
quantization of its angles.  Test infrastructure only: the CUDA library never imports this.

Source.
  [JJ] 第二部分 第一步 "PolarQuant——换一个坐标系来看数据": after the random rotation the vector is
       written as radius + angles: coordinates are paired and each pair turned into polar form,
       then the radii are paired and transformed again, recursively, until one final radius and
       a set of angles remain; the angle distributions are known after the rotation, so no
       per-block constants are stored.
  [VC] 第一階段 "PolarQuant（極座標量化）": a radius for the size, angles for the direction.

Definitions (R = reading where the pages are silent):
  y = (1/sqrt(d)) H (D x)      the rotation of oracle.rotation, x not normalised (d = 2^L)
  level 1:  r1_i = |(y_2i, y_2i+1)|,  a1_i = atan2(y_2i+1, y_2i) in (-pi, pi]
  level l:  rl_i = |(r_{l-1,2i}, r_{l-1,2i+1})|,  al_i = atan2(r_{l-1,2i+1}, r_{l-1,2i}) in [0, pi/2]
  the final radius r_L = ||x|| is the stored norm; there are d - 1 angles, ordered level 1 first
  (d/2 of them), then level 2, ..., level L (one) (R)
  angle laws for a direction uniform on the sphere (R: the standard hyperspherical-coordinate
  result the pages allude to): level 1 uniform on (-pi, pi]; level l >= 2, with k = 2^(l-1),
      f_l(a) = 2 (sin a cos a)^(k-1) / B(k/2, k/2)   on [0, pi/2]
  quantizer (R): b bits per angle at every level, so the budget matches b bits per coordinate;
  level 1: 2^b equal cells starting at -pi with the cell middles as centroids (the Lloyd-Max
  quantizer of the uniform law); levels >= 2: Lloyd-Max for f_l
  reconstruction, top down: r_{l-1,2i} = r_l,i cos(a^), r_{l-1,2i+1} = r_l,i sin(a^), then
  y^_2i = r_1,i cos(a^_1,i), y^_2i+1 = r_1,i sin(a^_1,i)
  QJL stage (the same as with the coordinate quantizer): r = y / ||x|| - y^ / ||x||, gamma = ||r||,
  bit_i = [(S r)_i >= 0]; score = ||x|| (<q', y^ / ||x||> + sqrt(pi/2)/m gamma <p, 2 bit - 1>)

Pinned by tests/test_oracle_polar.py: the laws integrate to 1 and match Monte-Carlo angles of
Gaussian vectors; Lloyd conditions by independent quadrature; the unquantized transform inverts
exactly and its final radius is the norm; a d = 8 brute force with explicit loops; the error
falls with b; the QJL-corrected score is unbiased over S.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from functools import lru_cache

import numpy as np
from scipy import integrate, special

from .rotation import rotate


def levels(d: int) -> int:
    if d < 2 or d & (d - 1):
        raise ValueError("d must be a power of two >= 2")
    return int(round(math.log2(d)))


def angle_density(a, level: int):
    """Density of a level-`level` angle of a uniformly random direction."""
    a = np.asarray(a, dtype=np.float64)
    if level == 1:
        return np.where((a > -math.pi) & (a <= math.pi), 1.0 / (2.0 * math.pi), 0.0)
    k = 2 ** (level - 1)
    inside = (a >= 0.0) & (a <= math.pi / 2)
    val = 2.0 * np.power(np.abs(np.sin(a) * np.cos(a)), k - 1) / special.beta(k / 2.0, k / 2.0)
    return np.where(inside, val, 0.0)


@lru_cache(maxsize=None)
def angle_codebook(level: int, bits: int, tol: float = 1e-13, max_iter: int = 100_000):
    """(centroids [2^b], thresholds [2^b - 1]) for the angles of one level."""
    L = 1 << bits
    if level == 1:
        w = 2.0 * math.pi / L
        edges = -math.pi + w * np.arange(L + 1)
        return 0.5 * (edges[:-1] + edges[1:]), edges[1:-1].copy()
    f = lambda a: float(angle_density(a, level))
    mass = lambda lo, hi: integrate.quad(f, lo, hi, epsabs=1e-14, epsrel=1e-13, limit=200)[0]
    mom = lambda lo, hi: integrate.quad(lambda a: a * f(a), lo, hi, epsabs=1e-14, epsrel=1e-13, limit=200)[0]
    # start from the quantiles of the law
    grid = np.linspace(0.0, math.pi / 2, 20001)
    cdf = np.concatenate([[0.0], np.cumsum(0.5 * (angle_density(grid[1:], level) + angle_density(grid[:-1], level))
                                           * np.diff(grid))])
    cdf /= cdf[-1]
    c = np.interp((np.arange(L) + 0.5) / L, cdf, grid)
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[0.0], t, [math.pi / 2]])
        new = np.array([mom(edges[i], edges[i + 1]) / mass(edges[i], edges[i + 1]) for i in range(L)])
        delta = np.max(np.abs(new - c))
        c = new
        if delta < tol:
            break
    return c, 0.5 * (c[:-1] + c[1:])


def transform(y):
    """y [n, d] -> (angles [n, d - 1] in the level order, final radius [n])."""
    y = np.asarray(y, dtype=np.float64)
    n, d = y.shape
    out = []
    a = np.arctan2(y[:, 1::2], y[:, 0::2])
    r = np.hypot(y[:, 0::2], y[:, 1::2])
    out.append(a)
    while r.shape[1] > 1:
        out.append(np.arctan2(r[:, 1::2], r[:, 0::2]))
        r = np.hypot(r[:, 0::2], r[:, 1::2])
    return np.concatenate(out, axis=1), r[:, 0]


def inverse(angles, radius, d: int):
    """(angles [n, d - 1], final radius [n]) -> y [n, d]."""
    angles = np.asarray(angles, dtype=np.float64)
    n = angles.shape[0]
    L = levels(d)
    # split the level blocks: level l has d / 2^l angles
    sizes = [d >> l for l in range(1, L + 1)]
    offs = np.concatenate([[0], np.cumsum(sizes)])
    r = np.asarray(radius, dtype=np.float64).reshape(n, 1)
    for l in range(L, 1, -1):
        a = angles[:, offs[l - 1]:offs[l]]
        nr = np.empty((n, 2 * r.shape[1]))
        nr[:, 0::2] = r * np.cos(a)
        nr[:, 1::2] = r * np.sin(a)
        r = nr
    a = angles[:, offs[0]:offs[1]]
    y = np.empty((n, d))
    y[:, 0::2] = r * np.cos(a)
    y[:, 1::2] = r * np.sin(a)
    return y


def level_of(d: int) -> np.ndarray:
    """Level of each of the d - 1 angle positions."""
    return np.concatenate([np.full(d >> l, l) for l in range(1, levels(d) + 1)])


def quantize_angles(angles, d: int, bits: int):
    """Angle codes [n, d - 1]: the count of the level's thresholds <= angle (R: a tie goes up)."""
    angles = np.asarray(angles, dtype=np.float64)
    lv = level_of(d)
    codes = np.zeros(angles.shape, dtype=np.int64)
    for l in np.unique(lv):
        _, t = angle_codebook(int(l), bits)
        sel = lv == l
        codes[:, sel] = np.sum(angles[:, sel, None] >= t[None, None, :], axis=2)
    return codes


def dequantize_angles(codes, d: int, bits: int):
    codes = np.asarray(codes, dtype=np.int64)
    lv = level_of(d)
    out = np.zeros(codes.shape)
    for l in np.unique(lv):
        c, _ = angle_codebook(int(l), bits)
        sel = lv == l
        out[:, sel] = c[codes[:, sel]]
    return out


@dataclass
class PolarEncoded:
    norm: np.ndarray      # [n]  ||x||
    codes: np.ndarray     # [n, d]  angle codes, position d - 1 unused (0)
    angles: np.ndarray    # [n, d - 1]  unquantized angles (for the threshold band of parity checks)
    yhat: np.ndarray      # [n, d]  reconstructed rotated unit vector
    rnorm: np.ndarray     # [n]
    bits: np.ndarray      # [n, m] QJL bits
    z: np.ndarray         # [n, m] QJL projections (for the sign band)


def encode(x, signs, S, bits: int) -> PolarEncoded:
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    y = rotate(x, signs)
    angles, radius = transform(y)
    codes = quantize_angles(angles, d, bits)
    nu = np.linalg.norm(x, axis=1)
    yhat = inverse(dequantize_angles(codes, d, bits), np.ones(n), d)  # unit radius
    safe = np.where(nu > 0, nu, 1.0)
    r = np.where(nu[:, None] > 0, y / safe[:, None], 0.0) - yhat
    S = np.asarray(S, dtype=np.float64)
    z = r @ S.T if S.shape[0] > 0 else np.zeros((n, 0))
    full = np.zeros((n, d), dtype=np.int64)
    full[:, :d - 1] = codes
    return PolarEncoded(norm=nu, codes=full, angles=angles, yhat=yhat, rnorm=np.linalg.norm(r, axis=1),
                        bits=(z >= 0).astype(np.uint8), z=z)


def reconstruct(norm, codes, signs, bits: int):
    """x^ = ||x|| D (1/sqrt d) H y^_unit from stored norms and angle codes [n, d]."""
    codes = np.asarray(codes, dtype=np.int64)
    n, d = codes.shape
    from .rotation import unrotate
    yhat = inverse(dequantize_angles(codes[:, :d - 1], d, bits), np.ones(n), d)
    return np.asarray(norm, dtype=np.float64)[:, None] * unrotate(yhat, signs)


def scores(qr, p, norm, codes, rnorm, qbits, bits: int):
    """Estimated inner products [nq, n] from prepared queries (oracle.estimate.prepare_query) and
    stored norms, angle codes, residual norms and QJL bits."""
    codes = np.asarray(codes, dtype=np.int64)
    n, d = codes.shape
    yhat = inverse(dequantize_angles(codes[:, :d - 1], d, bits), np.ones(n), d)
    mse = np.asarray(qr) @ yhat.T
    m = np.asarray(p).shape[1]
    if m > 0:
        pm = 2.0 * np.asarray(qbits, dtype=np.float64) - 1.0
        corr = math.sqrt(math.pi / 2.0) / m * np.asarray(rnorm, dtype=np.float64)[None, :] * (np.asarray(p) @ pm.T)
    else:
        corr = 0.0
    return np.asarray(norm, dtype=np.float64)[None, :] * (mse + corr)
