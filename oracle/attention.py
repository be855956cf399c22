"""Decode attention over the compressed KV cache (fp64), computed directly.

Source.
  [JJ] 第一部分 "KV 缓存是什么": during decoding each new token attends over the stored Key and
       Value vectors of all previous tokens.
  [JJ] 第三部分 "推理速度": attention logits are computed against the compressed keys and the
       computation is memory-bandwidth bound.
  [ZC] 第五部分 / 第六部分: values are compressed with the same quantizer (MSE stage only here)
       and dequantized inside the weighted sum.

Definitions (R = reading where the pages are silent):
  logits  l_t = scale * score(q, k_t)        scale = 1/sqrt(d) unless given (R)
  weights w   = softmax(l) over the sequence's tokens
  values  v^_t = nu_t * D_V (1/sqrt(d)) H c_V[code_t]      (inverse rotation of the centroids)
  output  o   = sum_t w_t v^_t
  grouped-query attention: query head hq reads KV head hq // (Hq / Hkv)  (R)
  an empty context gives o = 0 (R)

Sparse V ([ZC] 第六部分 "Sparse V Dequant"): the attention weights act as a gate, and value rows
whose weight is below a threshold tau (the pages use 1e-6) are not dequantized, i.e. they are left
out of the weighted sum; the softmax normalisation itself still covers every token (R: the pages
skip only the value decompression step):
  o = sum_{t : w_t >= tau} w_t v^_t
tau = 0 (the default) keeps every row.

Cache addressing: every packed array is indexed by a slot.
  contiguous: slot(b, h, t) = (b * Hkv + h) * ctx_stride + t
  paged:      slot(b, h, t) = (block_table[b, t // B] * Hkv + h) * B + t % B,  B = 16 tokens

This oracle reconstructs each value vector and sums in the original domain, one (batch, query
head) at a time; it does not split the context and does not work in the rotated domain.

Pinned by tests/test_oracle_attention.py: with m = 0 it equals plain softmax attention over the
reconstructed keys and values; softmax weights sum to 1; paged == contiguous on the same data;
grouped heads read the right KV head; empty contexts.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from . import polar
from .estimate import prepare_query, scores
from .rotation import unrotate


@dataclass
class Cache:
    """Unpacked cache arrays indexed by slot."""
    norm: np.ndarray            # [slots]
    codes: np.ndarray           # [slots, d]
    rnorm: np.ndarray = None    # [slots]     (keys with QJL)
    bits: np.ndarray = None     # [slots, m]  (keys with QJL)


def token_slots(b: int, h: int, length: int, n_kv: int, ctx_stride=None, block_table=None,
                block_tokens: int = 16) -> np.ndarray:
    t = np.arange(length, dtype=np.int64)
    if block_table is None:
        return (b * n_kv + h) * int(ctx_stride) + t
    blk = np.asarray(block_table, dtype=np.int64)[b, t // block_tokens]
    return (blk * n_kv + h) * block_tokens + t % block_tokens


def attend_decode(q, kcache: Cache, vcache: Cache, ctx_lens, n_kv: int,
                  k_signs, k_S, k_centroids, v_signs, v_centroids,
                  scale=None, ctx_stride=None, block_table=None, block_tokens: int = 16,
                  heads=None, sparse_v: float = 0.0, k_polar=None, v_polar=None):
    """q [B, Hq, d] -> o [B, Hq, d].  `heads` optionally restricts the (b, hq) pairs computed
    (others are left as NaN), for sampled checks at large sizes.  `sparse_v` is the Sparse V
    threshold tau on the softmax weights (0 = every value row is used).  `k_polar` / `v_polar`:
    the bits per angle when the keys / values carry PolarQuant angle codes (oracle.polar), whose
    scores and reconstructions then replace the coordinate codebook's."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    G = Hq // n_kv
    if scale is None or scale == 0:
        scale = 1.0 / math.sqrt(d)
    k_S = np.asarray(k_S, dtype=np.float64)
    out = np.full((B, Hq, d), np.nan)
    pairs = heads if heads is not None else [(b, hq) for b in range(B) for hq in range(Hq)]
    for b, hq in pairs:
        h = hq // G
        L = int(ctx_lens[b])
        if L == 0:
            out[b, hq] = 0.0
            continue
        sl = token_slots(b, h, L, n_kv, ctx_stride, block_table, block_tokens)
        qr, p = prepare_query(q[b, hq][None, :], k_signs, k_S)
        rn = kcache.rnorm[sl] if kcache.rnorm is not None else np.zeros(L)
        bt = kcache.bits[sl] if kcache.bits is not None else np.zeros((L, 0))
        if k_polar:
            s = polar.scores(qr, p, kcache.norm[sl], kcache.codes[sl], rn, bt, k_polar)[0]
        else:
            s = scores(qr, p, kcache.norm[sl], kcache.codes[sl], rn, bt, k_centroids)[0]
        logits = scale * s
        w = np.exp(logits - np.max(logits))
        w /= np.sum(w)
        keep = w >= sparse_v if sparse_v > 0 else np.ones(L, dtype=bool)
        if v_polar:
            vhat = polar.reconstruct(vcache.norm[sl][keep], vcache.codes[sl][keep], v_signs, v_polar)
        else:
            cv = np.asarray(v_centroids, dtype=np.float64)[vcache.codes[sl][keep]]
            vhat = vcache.norm[sl][keep][:, None] * unrotate(cv, v_signs)
        out[b, hq] = w[keep] @ vhat
    return out
