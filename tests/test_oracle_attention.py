"""Pins for oracle.attention: decode attention over the compressed cache.

Independent references: plain softmax attention (numpy) over keys and values reconstructed with
scipy's dense Hadamard matrix (with m = 0 the estimator is exactly <q, k^>), the paged layout
against the contiguous one, softmax normalisation, grouped-query head mapping, empty contexts,
and closeness to exact attention at 4 bits ([JJ] 第三部分: quality is kept at low bit widths).
"""
import math

import numpy as np
import pytest
from scipy.linalg import hadamard

from oracle import attention, codebook, encode


def _cache(x, D, S, c, t):
    e = encode.encode(x, D, S, c, t)
    return attention.Cache(norm=e.norm, codes=e.codes, rnorm=e.rnorm, bits=e.bits), e


def _recon(norm, codes, D, c):
    d = codes.shape[1]
    H = hadamard(d) / math.sqrt(d)
    return norm[:, None] * ((c[codes] @ H.T) * D)


def plain_attention(q, K, V, scale):
    logits = scale * (K @ q)
    w = np.exp(logits - logits.max())
    w /= w.sum()
    return w @ V


@pytest.mark.parametrize("d,kb,vb", [(16, 2, 3), (128, 3, 2)])
def test_mse_only_attention_equals_plain_softmax_attention(d, kb, vb):
    B, Hkv, G, ctx = 2, 2, 4, 40
    lens = [40, 23]
    rng = np.random.default_rng(d)
    K = rng.standard_normal((B * Hkv * ctx, d)) * rng.lognormal(size=d)
    V = rng.standard_normal((B * Hkv * ctx, d)) * rng.lognormal(size=d)
    Dk = rng.choice([-1.0, 1.0], size=d)
    Dv = rng.choice([-1.0, 1.0], size=d)
    ck, tk = codebook.codebook(d, kb)
    cv, tv = codebook.codebook(d, vb)
    kc, ke = _cache(K, Dk, np.zeros((0, d)), ck, tk)
    vc, ve = _cache(V, Dv, np.zeros((0, d)), cv, tv)
    q = rng.standard_normal((B, Hkv * G, d))
    out = attention.attend_decode(q, kc, vc, lens, Hkv, Dk, np.zeros((0, d)), ck, Dv, cv,
                                  ctx_stride=ctx)
    Kh = _recon(ke.norm, ke.codes, Dk, ck)
    Vh = _recon(ve.norm, ve.codes, Dv, cv)
    for b in range(B):
        for hq in range(Hkv * G):
            h = hq // G
            sl = slice((b * Hkv + h) * ctx, (b * Hkv + h) * ctx + lens[b])
            ref = plain_attention(q[b, hq], Kh[sl], Vh[sl], 1 / math.sqrt(d))
            np.testing.assert_allclose(out[b, hq], ref, rtol=1e-11, atol=1e-12)


def test_paged_equals_contiguous():
    d, bits, m = 32, 2, 32
    B, Hkv, G, blk = 3, 2, 2, 16
    lens = np.array([37, 16, 5])
    rng = np.random.default_rng(3)
    Dk = rng.choice([-1.0, 1.0], size=d)
    Dv = rng.choice([-1.0, 1.0], size=d)
    S = rng.standard_normal((m, d))
    ck, tk = codebook.codebook(d, bits)
    cv, tv = codebook.codebook(d, 3)
    ctx = 48
    K = rng.standard_normal((B * Hkv * ctx, d))
    V = rng.standard_normal((B * Hkv * ctx, d))
    kc, _ = _cache(K, Dk, S, ck, tk)
    vc, _ = _cache(V, Dv, np.zeros((0, d)), cv, tv)
    q = rng.standard_normal((B, Hkv * G, d))
    ref = attention.attend_decode(q, kc, vc, lens, Hkv, Dk, S, ck, Dv, cv, ctx_stride=ctx)
    # scatter the same tokens into shuffled 16-token blocks
    nblk = [(int(n) + blk - 1) // blk for n in lens]
    perm = rng.permutation(sum(nblk) + 3)          # a few unused blocks too
    table = np.zeros((B, max(nblk)), dtype=np.int64)
    o = 0
    for b in range(B):
        table[b, :nblk[b]] = perm[o:o + nblk[b]]
        o += nblk[b]
    nslots = (sum(nblk) + 3) * Hkv * blk

    def scatter(cache, with_qjl):
        out = attention.Cache(norm=np.zeros(nslots), codes=np.zeros((nslots, d), dtype=np.int64))
        if with_qjl:
            out.rnorm = np.zeros(nslots)
            out.bits = np.zeros((nslots, m), dtype=np.uint8)
        for b in range(B):
            for h in range(Hkv):
                src = attention.token_slots(b, h, int(lens[b]), Hkv, ctx_stride=ctx)
                dst = attention.token_slots(b, h, int(lens[b]), Hkv, block_table=table)
                out.norm[dst] = cache.norm[src]
                out.codes[dst] = cache.codes[src]
                if with_qjl:
                    out.rnorm[dst] = cache.rnorm[src]
                    out.bits[dst] = cache.bits[src]
        return out

    got = attention.attend_decode(q, scatter(kc, True), scatter(vc, False), lens, Hkv, Dk, S, ck,
                                  Dv, cv, block_table=table)
    np.testing.assert_array_equal(got, ref)


def test_empty_context_gives_zero():
    d = 16
    rng = np.random.default_rng(0)
    D = rng.choice([-1.0, 1.0], size=d)
    c, t = codebook.codebook(d, 2)
    kc, _ = _cache(rng.standard_normal((16, d)), D, np.zeros((0, d)), c, t)
    out = attention.attend_decode(rng.standard_normal((2, 1, d)), kc, kc, [0, 8], 1, D,
                                  np.zeros((0, d)), c, D, c, ctx_stride=8)
    assert np.all(out[0, 0] == 0.0) and np.all(np.isfinite(out[1, 0]))


def test_single_token_returns_its_value():
    # softmax over one token is 1, so the output is that token's reconstructed value.
    d = 32
    rng = np.random.default_rng(1)
    D = rng.choice([-1.0, 1.0], size=d)
    c, t = codebook.codebook(d, 3)
    kc, _ = _cache(rng.standard_normal((1, d)), D, rng.standard_normal((32, d)), c, t)
    vc, ve = _cache(rng.standard_normal((1, d)), D, np.zeros((0, d)), c, t)
    out = attention.attend_decode(rng.standard_normal((1, 1, d)), kc, vc, [1], 1, D,
                                  rng.standard_normal((32, d)), c, D, c, ctx_stride=1)
    np.testing.assert_allclose(out[0, 0], _recon(ve.norm, ve.codes, D, c)[0], atol=1e-12)


def test_four_bit_attention_is_close_to_exact():
    d, ctx = 128, 512
    rng = np.random.default_rng(2)
    K = rng.standard_normal((ctx, d))
    V = rng.standard_normal((ctx, d))
    Dk = rng.choice([-1.0, 1.0], size=d)
    Dv = rng.choice([-1.0, 1.0], size=d)
    S = rng.standard_normal((d, d))
    ck, tk = codebook.codebook(d, 3)
    cv, tv = codebook.codebook(d, 4)
    kc, _ = _cache(K, Dk, S, ck, tk)
    vc, _ = _cache(V, Dv, np.zeros((0, d)), cv, tv)
    q = rng.standard_normal((1, 1, d)) * 0.5
    out = attention.attend_decode(q, kc, vc, [ctx], 1, Dk, S, ck, Dv, cv, ctx_stride=ctx)[0, 0]
    ref = plain_attention(q[0, 0], K, V, 1 / math.sqrt(d))
    # a sanity bound only: the QJL term is unbiased but noisy, so sharp softmaxes amplify it
    assert np.linalg.norm(out - ref) < 0.25 * np.linalg.norm(ref)


def _small_case(seed, d=16, ctx=60, kb=2, vb=3, spread=8.0):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((ctx, d)) * spread
    V = rng.standard_normal((ctx, d))
    Dk = rng.choice([-1.0, 1.0], size=d)
    Dv = rng.choice([-1.0, 1.0], size=d)
    ck, tk = codebook.codebook(d, kb)
    cv, tv = codebook.codebook(d, vb)
    kc, ke = _cache(K, Dk, np.zeros((0, d)), ck, tk)
    vc, ve = _cache(V, Dv, np.zeros((0, d)), cv, tv)
    q = rng.standard_normal((1, 1, d)) * spread
    return q, kc, ke, vc, ve, Dk, Dv, ck, cv


def test_sparse_v_threshold_zero_is_plain_attention():
    q, kc, ke, vc, ve, Dk, Dv, ck, cv = _small_case(5)
    a = attention.attend_decode(q, kc, vc, [60], 1, Dk, np.zeros((0, 16)), ck, Dv, cv, ctx_stride=60)
    b = attention.attend_decode(q, kc, vc, [60], 1, Dk, np.zeros((0, 16)), ck, Dv, cv, ctx_stride=60,
                                sparse_v=0.0)
    np.testing.assert_array_equal(a, b)


def test_sparse_v_drops_exactly_the_rows_below_the_threshold():
    """Hand-built gate: the rows whose softmax weight (over all tokens, normalisation unchanged)
    is below tau are left out of the sum, every other row is kept with its full weight."""
    d, ctx = 16, 60
    q, kc, ke, vc, ve, Dk, Dv, ck, cv = _small_case(6)
    Kh = _recon(ke.norm, ke.codes, Dk, ck)
    Vh = _recon(ve.norm, ve.codes, Dv, cv)
    logits = (Kh @ q[0, 0]) / math.sqrt(d)
    w = np.exp(logits - logits.max())
    w /= w.sum()
    order = np.sort(w)
    tau = 0.5 * (order[20] + order[21])  # a threshold between the 21st and 22nd smallest weights
    dropped = w < tau
    assert dropped.sum() == 21
    expect = (w * ~dropped) @ Vh
    got = attention.attend_decode(q, kc, vc, [ctx], 1, Dk, np.zeros((0, d)), ck, Dv, cv, ctx_stride=ctx,
                                  sparse_v=tau)[0, 0]
    np.testing.assert_allclose(got, expect, rtol=1e-11, atol=1e-12)
    # the dropped mass is what changes: |o - o_sparse| <= sum of dropped weights x max |v^|
    full = attention.attend_decode(q, kc, vc, [ctx], 1, Dk, np.zeros((0, d)), ck, Dv, cv, ctx_stride=ctx)[0, 0]
    assert np.max(np.abs(full - got)) <= w[dropped].sum() * np.max(np.abs(Vh)) + 1e-15
    # a threshold above every weight leaves nothing; one at or below the smallest keeps all
    none = attention.attend_decode(q, kc, vc, [ctx], 1, Dk, np.zeros((0, d)), ck, Dv, cv, ctx_stride=ctx,
                                   sparse_v=1.01)[0, 0]
    np.testing.assert_array_equal(none, np.zeros(d))
    allk = attention.attend_decode(q, kc, vc, [ctx], 1, Dk, np.zeros((0, d)), ck, Dv, cv, ctx_stride=ctx,
                                   sparse_v=order[0])[0, 0]
    np.testing.assert_allclose(allk, full, rtol=1e-12, atol=1e-14)
