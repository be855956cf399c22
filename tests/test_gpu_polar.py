"""GPU parity of the PolarQuant first stage (tq_ctx_create_polar; "谷歌 TurboQuant 深度拆解" 第二部分
第一步: recursive polar transform of the rotated vector, angles quantized with the Lloyd-Max
codebooks of their levels' known laws) against oracle.polar.

Angle codes are compared like the coordinate codes: bit-exact except where the angle lies within
1e-5 of a threshold of its level (fp32 atan2 against fp64), at most 1e-4 of the entries; norms,
residual norms (rows without a flip) and QJL signs (|z| band) as for the coordinate quantizer.
Scores are checked stage-isolated: the oracle scores the library's own packed bytes.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import encode as oenc
from oracle import estimate as oest
from oracle import polar
from parity import BAND, MAX_FLIP_FRACTION, assert_scores_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_06_b200 import tq as _tq
    return _tq


def _ctx(tq, bits, m, seed):
    d = 128
    D = synth.rotation_signs(d, seed)
    S = synth.qjl_matrix(m, d, seed + 1) if m else None
    return tq.Context(d, bits, m, D, S, polar=True), D.double().numpy(), (S.double().numpy() if m else np.zeros((0, d)))


def _near_threshold(angles, d, bits):
    lv = polar.level_of(d)
    near = np.zeros(angles.shape, dtype=bool)
    for l in np.unique(lv):
        _, t = polar.angle_codebook(int(l), bits)
        sel = lv == l
        near[:, sel] = np.min(np.abs(angles[:, sel, None] - t[None, None, :]), axis=2) < BAND
    return near


@pytest.mark.parametrize("bits,m", [(1, 0), (2, 128), (3, 128), (4, 0), (2, 64)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_polar_encode_matches_oracle(tq, bits, m, dtype):
    d, n = 128, 3001
    ctx, D, S = _ctx(tq, bits, m, 300 + 10 * bits + m)
    x = (torch.randn(n, d, generator=torch.Generator().manual_seed(bits)) *
         torch.exp(torch.randn(d, generator=torch.Generator().manual_seed(3)))).to(dtype)
    packed = tq.Packed.allocate(ctx, n)
    tq.encode_kv(ctx, x.cuda(), packed)
    torch.cuda.synchronize()
    enc = polar.encode(x.double().numpy(), D, S, bits)
    codes = oenc.unpack_codes(packed.codes.cpu().numpy(), d, bits)
    np.testing.assert_allclose(packed.norm.double().cpu().numpy(), enc.norm, rtol=2e-6)
    bad = codes[:, :d - 1] != enc.codes[:, :d - 1]
    near = _near_threshold(enc.angles, d, bits)
    assert not np.any(bad & ~near), "angle code mismatch outside the threshold band"
    assert bad.sum() <= max(1, MAX_FLIP_FRACTION * bad.size), bad.sum()
    assert np.all(codes[:, d - 1] == 0)
    if m:
        rows_ok = ~bad.any(axis=1)
        np.testing.assert_allclose(packed.rnorm.double().cpu().numpy()[rows_ok], enc.rnorm[rows_ok], rtol=2e-5,
                                   atol=1e-6)
        sb = oenc.unpack_signs(packed.signs.cpu().numpy(), m)
        sbad = (sb != enc.bits) & rows_ok[:, None]
        assert not np.any(sbad & ~(np.abs(enc.z) < BAND)), "sign mismatch outside the |z| band"


@pytest.mark.parametrize("bits,m", [(2, 128), (3, 0)])
def test_polar_scores_match_oracle(tq, bits, m):
    """The Tiny workload's keys with the PolarQuant first stage: scores of 8 queries."""
    keys, queries = synth.tiny(seed=0)
    ctx, D, S = _ctx(tq, bits, m, 340 + bits)
    packed = tq.Packed.allocate(ctx, keys.shape[0])
    tq.encode_kv(ctx, keys.cuda(), packed)
    got = tq.scores(ctx, queries.cuda(), packed).cpu().numpy()
    d = 128
    codes = oenc.unpack_codes(packed.codes.cpu().numpy(), d, bits)
    sb = oenc.unpack_signs(packed.signs.cpu().numpy(), m) if m else np.zeros((keys.shape[0], 0))
    rn = packed.rnorm.double().cpu().numpy() if m else np.zeros(keys.shape[0])
    qr, p = oest.prepare_query(queries.double().numpy(), D, S)
    ref = polar.scores(qr, p, packed.norm.double().cpu().numpy(), codes, rn, sb, bits)
    assert_scores_close(got, ref)


@pytest.mark.parametrize("bits,m,k", [(2, 128, 10), (3, 0, 40)])
def test_polar_search_topk(tq, bits, m, k):
    """PolarQuant database through the CUDA-core scans (k <= 32 and the large-k scan), against the
    oracle's PolarQuant scores of the library's own bytes."""
    from oracle import search as osearch
    from parity import assert_topk_equivalent
    n, d = 3001, 128
    ctx, D, S = _ctx(tq, bits, m, 360 + bits)
    X = synth.unit_rows(n, d, seed=11) * 2.0
    packed = tq.Packed.allocate(ctx, n)
    tq.encode_kv(ctx, X.cuda(), packed)
    for nq in (5, 40):
        Q = synth.unit_rows(nq, d, seed=12 + nq)
        s, i = tq.search_topk(ctx, Q.cuda(), packed, k)
        codes = oenc.unpack_codes(packed.codes.cpu().numpy(), d, bits)
        sb = oenc.unpack_signs(packed.signs.cpu().numpy(), m) if m else np.zeros((n, 0))
        rn = packed.rnorm.double().cpu().numpy() if m else np.zeros(n)
        qr, p = oest.prepare_query(Q.double().numpy(), D, S)
        ref_full = polar.scores(qr, p, packed.norm.double().cpu().numpy(), codes, rn, sb, bits)
        ref_s, _ = osearch.topk(ref_full, k)
        assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)


@pytest.mark.parametrize("kpolar,vpolar", [(True, True), (True, False), (False, True)])
def test_polar_attention(tq, kpolar, vpolar):
    """Decode attention with PolarQuant keys and/or values (the general path), paged and ragged,
    GQA 4, against the oracle evaluated on the library's own bytes."""
    from oracle import attention as oattn
    from oracle import codebook as ocb
    from parity import assert_attention_close
    d, hkv, group, lens, bits_k, bits_v = 128, 2, 4, [300, 17, 513], 2, 3
    batch = len(lens)
    DK, DV = synth.rotation_signs(d, 401), synth.rotation_signs(d, 402)
    SK = synth.qjl_matrix(128, d, 403)
    kctx = tq.Context(d, bits_k, 128, DK, SK, polar=kpolar)
    vctx = tq.Context(d, bits_v, 0, DV, polar=vpolar)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    table, nblocks = synth.shuffled_block_table(lens_t, seed=404)
    cap = nblocks * hkv * synth.BLOCK_TOKENS
    K = synth.channel_scaled(batch, hkv, max(lens), d, seed=405)
    V = synth.channel_scaled(batch, hkv, max(lens), d, seed=406)
    kp, vp = tq.Packed.allocate(kctx, cap), tq.Packed.allocate(vctx, cap)
    for b in range(batch):
        for h in range(hkv):
            sl = torch.as_tensor(oattn.token_slots(b, h, lens[b], hkv, block_table=table.numpy()), dtype=torch.int64)
            tq.encode_kv(kctx, K[b, h, :lens[b]].cuda(), kp, slots=sl.cuda())
            tq.encode_kv(vctx, V[b, h, :lens[b]].cuda(), vp, slots=sl.cuda())
    q = synth.decode_queries(batch, hkv * group, d, seed=407, dtype=torch.bfloat16)
    out = tq.attend_decode(kctx, vctx, q.cuda(), kp, vp, lens_t.cuda(), max(lens), n_kv_heads=hkv,
                           block_table=table.cuda(), block_size=synth.BLOCK_TOKENS)
    torch.cuda.synchronize()
    kcache = oattn.Cache(norm=kp.norm.double().cpu().numpy(), codes=oenc.unpack_codes(kp.codes.cpu().numpy(), d, bits_k),
                         rnorm=kp.rnorm.double().cpu().numpy(), bits=oenc.unpack_signs(kp.signs.cpu().numpy(), 128))
    vcache = oattn.Cache(norm=vp.norm.double().cpu().numpy(), codes=oenc.unpack_codes(vp.codes.cpu().numpy(), d, bits_v))
    ck, _ = ocb.codebook(d, bits_k)
    cv, _ = ocb.codebook(d, bits_v)
    ref = oattn.attend_decode(q.double().numpy(), kcache, vcache, lens, hkv, DK.double().numpy(), SK.double().numpy(), ck,
                              DV.double().numpy(), cv, block_table=table.numpy(),
                              k_polar=bits_k if kpolar else None, v_polar=bits_v if vpolar else None)
    assert_attention_close(out.cpu().numpy(), ref)
    assert tq.device_status() == 0
