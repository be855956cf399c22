"""Encode: norm -> rotate -> Lloyd-Max codes -> residual -> QJL sign sketch (fp64), and the
packed byte layout.

Source.
  [JJ] 第一部分 "传统量化为什么不够用" and [VC] 零元數據: no per-block scale or zero-point is
       stored; the only per-vector scalar of the first stage is the vector's norm.
  [JJ] 第二部分 第一步 (PolarQuant): random rotation, then a fixed optimal scalar quantizer per
       rotated coordinate (the coordinate law is known, see oracle.codebook).
  [JJ] 第二部分 第二步 (QJL) and [VC] 第二階段: the residual of the first stage is projected
       with a Johnson-Lindenstrauss matrix and only the sign of each projected coordinate is
       kept (1 bit each).
  [LP] 二.2: the standard JL matrix has iid N(0,1) entries; the same section gives the fast
       (FJLT, y = P H D x) and sparse (Achlioptas) alternatives.  `srht_matrix` builds the
       structured one used as an option here: S = P H D2.
  [LP] 二.4 "CUDA/GPU 优化": codes are bit-packed into machine words.

Definitions (readings where the pages are silent are marked R):
  nu    = ||x||_2                                         (stored, fp32 on the GPU)
  u     = x / nu, and u = 0 when nu = 0                   (R: quantize the unit vector)
  y     = (1/sqrt(d)) H (D u)                             (oracle.rotation)
  code  = #{ i : t_i <= y_j }                              (R: a tie goes to the upper cell)
  r     = y - c[code],   gamma = ||r||_2                  (R: residual in the rotated domain)
  z     = S r,  bit_i = 1 if z_i >= 0 else 0              (R: sign(0) = +1)

Packed layout (R; the pages only say "bit-packing").  Every vector owns:
  codes: `code_bytes(d, b)` bytes = b bit-planes of d bits each, padded to a multiple of 16 B.
         Bit t of code_j lives in byte (t*d + j) // 8, bit (t*d + j) % 8 (LSB first).
  signs: `sign_bytes(m)` bytes; bit i lives in byte i // 8, bit i % 8, padded to 16 B.
  norm, rnorm: one fp32 each, in separate arrays.

Pinned by tests/test_oracle_encode.py (brute force at d=8 with the dense Hadamard matrix, a
dense S and an argmin over all levels; a hand-written packing example; round trips).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .rotation import rotate, sylvester


def code_bytes(d: int, bits: int) -> int:
    raw = (bits * d + 7) // 8
    return (raw + 15) // 16 * 16


def sign_bytes(m: int) -> int:
    if m == 0:
        return 0
    return ((m + 7) // 8 + 15) // 16 * 16


def quantize(y, thresholds) -> np.ndarray:
    """code = number of thresholds <= y (a value equal to a threshold goes to the upper cell)."""
    y = np.asarray(y, dtype=np.float64)
    t = np.asarray(thresholds, dtype=np.float64)
    return np.sum(y[..., None] >= t, axis=-1).astype(np.int64)


@dataclass
class Encoded:
    norm: np.ndarray      # [n]       ||x||
    codes: np.ndarray     # [n, d]    int codes in [0, 2^b)
    rnorm: np.ndarray     # [n]       ||r|| (zeros when m == 0)
    bits: np.ndarray      # [n, m]    0/1 sign bits
    y: np.ndarray         # [n, d]    pre-quantization rotated unit vector
    z: np.ndarray         # [n, m]    pre-sign projection S r


def encode(x, signs, S, centroids, thresholds) -> Encoded:
    """Encode rows of x ([n, d]) with rotation signs D ([d]), JL matrix S ([m, d], m may be 0)
    and a codebook (centroids [L], thresholds [L-1])."""
    x = np.asarray(x, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    t = np.asarray(thresholds, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    n, d = x.shape
    norm = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(norm > 0.0, norm, 1.0)
    u = np.where(norm[:, None] > 0.0, x / safe[:, None], 0.0)
    y = rotate(u, signs)
    codes = quantize(y, t)
    r = y - c[codes]
    m = S.shape[0]
    if m > 0:
        rnorm = np.sqrt(np.sum(r * r, axis=1))
        z = r @ S.T
        bits = (z >= 0.0).astype(np.uint8)
    else:
        rnorm = np.zeros(n)
        z = np.zeros((n, 0))
        bits = np.zeros((n, 0), dtype=np.uint8)
    return Encoded(norm=norm, codes=codes, rnorm=rnorm, bits=bits, y=y, z=z)


def store_norms(enc: Encoded, norm_bits: int = 32) -> Encoded:
    """The encoding as stored: with norm_bits = 16 the norms ||x|| and gamma are kept in IEEE half
    precision (round to nearest even, values above the largest half 65504 kept as 65504), the only
    per-vector constants being quantization metadata kept in FP16 or FP32 ([JJ] 第一部分)
    (reading: the option saves 4 bytes per vector with a QJL stage).  Codes and signs are unchanged
    (they come from the exact norm)."""
    if norm_bits == 32:
        return enc
    if norm_bits != 16:
        raise ValueError("norm_bits must be 32 or 16")
    h = lambda a: np.minimum(np.asarray(a, dtype=np.float64), 65504.0).astype(np.float16).astype(np.float64)
    return Encoded(**{**enc.__dict__, "norm": h(enc.norm), "rnorm": h(enc.rnorm)})


def pack_codes(codes, bits: int) -> np.ndarray:
    """[n, d] codes -> [n, code_bytes] uint8, plane-major LSB-first."""
    codes = np.asarray(codes, dtype=np.int64)
    n, d = codes.shape
    stream = np.zeros((n, code_bytes(d, bits) * 8), dtype=np.uint8)
    for t in range(bits):
        stream[:, t * d:(t + 1) * d] = (codes >> t) & 1
    return np.packbits(stream, axis=1, bitorder="little")


def unpack_codes(buf, d: int, bits: int) -> np.ndarray:
    """[n, code_bytes] uint8 -> [n, d] codes (inverse of pack_codes)."""
    buf = np.asarray(buf, dtype=np.uint8)
    stream = np.unpackbits(buf, axis=1, bitorder="little").astype(np.int64)
    codes = np.zeros((buf.shape[0], d), dtype=np.int64)
    for t in range(bits):
        codes |= stream[:, t * d:(t + 1) * d] << t
    return codes


def pack_signs(bits_) -> np.ndarray:
    """[n, m] 0/1 -> [n, sign_bytes] uint8, LSB-first."""
    bits_ = np.asarray(bits_, dtype=np.uint8)
    n, m = bits_.shape
    stream = np.zeros((n, sign_bytes(m) * 8), dtype=np.uint8)
    stream[:, :m] = bits_
    return np.packbits(stream, axis=1, bitorder="little")


def unpack_signs(buf, m: int) -> np.ndarray:
    buf = np.asarray(buf, dtype=np.uint8)
    return np.unpackbits(buf, axis=1, bitorder="little")[:, :m].astype(np.uint8)


# ---------------------------------------------------------------- token-block layout for values
# Reading (the pages only say "bit-packing"): for attention values the codes of 16 consecutive
# slots may be stored token-transposed.  Block k = slots 16k..16k+15 owns 16 * code_bytes bytes,
# read as little-endian 32-bit words W:
#   W[q*d + j] (q < b//2):    bit t = bit 2q of code_j of slot 16k+t, bit 16+t = bit 2q+1
#   W[(b//2)*d + j//2] (b odd): bit 16*(j%2) + t = bit b-1 of code_j of slot 16k+t
def pack_codes_block16(codes, bits: int) -> np.ndarray:
    """[n, d] codes (n a multiple of 16) -> [n, code_bytes] uint8 in the token-block layout."""
    codes = np.asarray(codes, dtype=np.int64)
    n, d = codes.shape
    if n % 16:
        raise ValueError("the token-block layout needs a multiple of 16 slots")
    cb = code_bytes(d, bits)
    nb = n // 16
    words = np.zeros((nb, 16 * cb // 4), dtype=np.uint64)
    blk = codes.reshape(nb, 16, d)                      # [block, token, j]
    tok = np.arange(16, dtype=np.uint64)[None, :, None]
    for q in range(bits // 2):
        lo = ((blk >> (2 * q)) & 1).astype(np.uint64) << tok
        hi = ((blk >> (2 * q + 1)) & 1).astype(np.uint64) << (tok + np.uint64(16))
        words[:, q * d:(q + 1) * d] = np.bitwise_or.reduce(lo | hi, axis=1)
    if bits % 2:
        j = np.arange(d)
        sh = (np.uint64(16) * (j % 2).astype(np.uint64))[None, None, :] + tok
        v = ((blk >> (bits - 1)) & 1).astype(np.uint64) << sh           # [block, token, j]
        per_j = np.bitwise_or.reduce(v, axis=1)                         # [block, j]
        base = (bits // 2) * d
        words[:, base:base + d // 2] = per_j[:, 0::2] | per_j[:, 1::2]
    return words.astype(np.uint32).view(np.uint8).reshape(n, cb)


def unpack_codes_block16(buf, d: int, bits: int) -> np.ndarray:
    """[n, code_bytes] uint8 in the token-block layout -> [n, d] codes."""
    buf = np.ascontiguousarray(np.asarray(buf, dtype=np.uint8))
    n, cb = buf.shape
    nb = n // 16
    words = buf.reshape(nb, 16 * cb).view(np.uint32).astype(np.int64)   # [block, words]
    tok = np.arange(16)[None, :, None]
    codes = np.zeros((nb, 16, d), dtype=np.int64)
    for q in range(bits // 2):
        w = words[:, None, q * d:(q + 1) * d]
        codes |= ((w >> tok) & 1) << (2 * q)
        codes |= ((w >> (tok + 16)) & 1) << (2 * q + 1)
    if bits % 2:
        j = np.arange(d)
        base = (bits // 2) * d
        w = words[:, None, base + j // 2]                                 # [block, 1, j]
        codes |= ((w >> (16 * (j % 2)[None, None, :] + tok)) & 1) << (bits - 1)
    return codes.reshape(n, d)


def srht_matrix(qjl_signs, m: int) -> np.ndarray:
    """Structured QJL matrix ([LP] 二.2, the fast JL transform y = P H D x): S = P H D2, with
    H the d x d Sylvester Hadamard matrix left unnormalised (entries +-1), D2 a diagonal of random
    signs (drawn independently of the rotation's D) and P keeping the first m rows (R: the random
    signs supply the randomness, so the kept rows are fixed).  S[i, j] = H[i, j] * D2[j]: entries
    +-1, unit variance like N(0,1) draws, and the rows are orthogonal.  The estimator keeps the
    Gaussian scale sqrt(pi/2)/m; it is unbiased over D2 to within Monte-Carlo resolution (exactly
    unbiased only for Gaussian rows)."""
    D2 = np.asarray(qjl_signs, dtype=np.float64)
    d = D2.shape[0]
    if not 0 < m <= d:
        raise ValueError("m must be in [1, d]")
    return sylvester(d)[:m] * D2[None, :]
