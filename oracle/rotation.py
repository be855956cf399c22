"""Randomized Walsh-Hadamard rotation (fp64).

Source.
  [LP] 二.2 "Johnson-Lindenstrauss 实现技术" (Fast JL, Ailon-Chazelle): y = P H D x with D a
       diagonal of random signs and H a Hadamard matrix.  Here P is the identity (no
       subsampling): the rotation keeps all d coordinates.
  [LP] 三.1 "线性代数": an orthogonal matrix preserves norms; H_n = H_1 (x) H_{n-1} (Sylvester).
  [JJ] 第二部分 第一步 "随机旋转" and [ZC] 第二部分 (Walsh-Hadamard): a random rotation is applied to
       every vector before quantization.

Definition used: y = (1/sqrt(d)) * H_d * (D * u), with H_d the d x d Sylvester Hadamard matrix
(entries (-1)^popcount(i & j)), so that the map is orthogonal.  Its inverse is
u = D * (1/sqrt(d)) * H_d * y (H_d is symmetric and H_d H_d = d I).

Pinned by tests/test_oracle_rotation.py: FWHT equals the dense product with scipy's Hadamard
matrix, H H^T = d I, and the rotation preserves norms to 1e-12 and inverts exactly.
"""
from __future__ import annotations

import math

import numpy as np


def sylvester(d: int) -> np.ndarray:
    """Dense Sylvester Hadamard matrix by the Kronecker recursion H_2n = H_2 (x) H_n."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    h2 = np.array([[1.0, 1.0], [1.0, -1.0]])
    while h.shape[0] < d:
        h = np.kron(h2, h)
    return h


def fwht(a: np.ndarray) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform along the last axis: returns a @ H_d."""
    a = np.array(a, dtype=np.float64, copy=True)
    d = a.shape[-1]
    if d & (d - 1):
        raise ValueError("length must be a power of two")
    h = 1
    while h < d:
        v = a.reshape(a.shape[:-1] + (d // (2 * h), 2, h))
        x = v[..., 0, :].copy()
        y = v[..., 1, :].copy()
        v[..., 0, :] = x + y
        v[..., 1, :] = x - y
        h *= 2
    return a


def rotate(u: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """y = (1/sqrt(d)) H (D u) along the last axis."""
    d = u.shape[-1]
    return fwht(np.asarray(u, dtype=np.float64) * np.asarray(signs, dtype=np.float64)) / math.sqrt(d)


def unrotate(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """u = D (1/sqrt(d)) H y along the last axis (inverse of `rotate`)."""
    d = y.shape[-1]
    return np.asarray(signs, dtype=np.float64) * fwht(y) / math.sqrt(d)
