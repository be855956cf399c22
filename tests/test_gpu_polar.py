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


def test_polar_rejects_attention_and_search(tq):
    ctx, D, S = _ctx(tq, 2, 128, 350)
    packed = tq.Packed.allocate(ctx, 64)
    with pytest.raises(tq.TqError) as e:
        tq.search_topk(ctx, torch.randn(3, 128).cuda(), packed, 4)
    assert e.value.status == 2
