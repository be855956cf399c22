"""GPU parity of Sparse V ("TurboQuant+ 深度解析" 第六部分: value rows whose softmax weight is below a
threshold are not dequantized) on the tensor-core decode path, against the oracle's Sparse V
(exact final weights, normalisation over every token).

The kernel decides with a running bound on each row's weight that is never below its final
weight, so it drops a subset of the rows the oracle drops; the rows it keeps in addition carry
weights below the threshold each.  The checks use a sharpened softmax (a larger logit scale) so
that a large share of the rows falls below 1e-6, at a Llama-8B layer length and on a ragged paged
batch."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oattn
from parity import Quantizer, assert_attention_close, oracle_cache, unpack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_06_b200 import tq as _tq
    return _tq


def _oracle(kq, vq, kp, vp, q, pairs, lens, slots_fn, group, scale, tau):
    out = {}
    for b, hq in pairs:
        h = hq // group
        L = int(lens[b])
        sl = np.asarray(slots_fn(b, h, L), dtype=np.int64)
        kc = oracle_cache(kq, *unpack(kq, kp, rows=sl))
        vc = oracle_cache(vq, *unpack(vq, vp, rows=sl))
        qq = q[b, hq][None, None].double().cpu().numpy()
        out[(b, hq)] = oattn.attend_decode(qq, kc, vc, [L], 1, kq.D64, kq.S64, kq.c, vq.D64, vq.c, scale=scale,
                                           ctx_stride=L, sparse_v=tau)[0, 0]
    return out


def _case(tq, paged, seed):
    d, hkv, group = 128, 2, 4
    kq = Quantizer(d, 2, d, seed=seed)
    vq = Quantizer(d, 3, 0, seed=seed + 1, layout=1)
    lens = [4096, 1500, 37] if paged else [4096]
    B = len(lens)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    maxlen = max(lens)
    if paged:
        table, nblocks = synth.shuffled_block_table(lens_t, seed=seed + 2)
        tab = table.numpy()
        cap = nblocks * hkv * 16
        slots_fn = lambda b, h, L: oattn.token_slots(b, h, L, hkv, block_table=tab)
    else:
        table = None
        cap = B * hkv * maxlen
        slots_fn = lambda b, h, L: oattn.token_slots(b, h, L, hkv, ctx_stride=maxlen)
    kp, vp = tq.Packed.allocate(kq.ctx, cap), tq.Packed.allocate(vq.ctx, cap)
    K = synth.channel_scaled(B, hkv, maxlen, d, seed=seed + 3)
    V = synth.channel_scaled(B, hkv, maxlen, d, seed=seed + 4)
    for b in range(B):
        for h in range(hkv):
            sl = torch.as_tensor(slots_fn(b, h, lens[b]), dtype=torch.int64).cuda()
            tq.encode_kv(kq.ctx, K[b, h, :lens[b]].cuda(), kp, slots=sl)
            tq.encode_kv(vq.ctx, V[b, h, :lens[b]].cuda(), vp, slots=sl)
    q = synth.decode_queries(B, hkv * group, d, seed=seed + 5)
    return kq, vq, kp, vp, q, lens, lens_t.cuda(), maxlen, table, slots_fn, hkv, group


@pytest.mark.parametrize("paged", [False, True])
def test_sparse_v_matches_oracle(tq, paged):
    kq, vq, kp, vp, q, lens, lens_g, maxlen, table, slots_fn, hkv, group = _case(tq, paged, 500 + int(paged))
    scale = 4.0 / np.sqrt(128.0)  # sharper than 1/sqrt(d): most weights fall far below 1e-6
    tau = 1e-6
    kw = dict(n_kv_heads=hkv, scale=scale, ctx_stride=None if paged else maxlen,
              block_table=None if table is None else table.cuda())
    dense = tq.attend_decode(kq.ctx, vq.ctx, q.cuda(), kp, vp, lens_g, maxlen, **kw)
    desc = tq.make_attn_desc(kq.ctx, vq.ctx, tuple(q.shape), kp, vp, lens_g, maxlen, sparse_v=tau, **kw)
    sparse = tq.attend_decode(kq.ctx, vq.ctx, q.cuda(), kp, vp, lens_g, maxlen, n_kv_heads=hkv, desc=desc)
    desc0 = tq.make_attn_desc(kq.ctx, vq.ctx, tuple(q.shape), kp, vp, lens_g, maxlen, sparse_v=0.0, **kw)
    zero = tq.attend_decode(kq.ctx, vq.ctx, q.cuda(), kp, vp, lens_g, maxlen, n_kv_heads=hkv, desc=desc0)
    torch.cuda.synchronize()
    assert tq.device_status() == 0
    assert torch.equal(zero, dense), "threshold 0 is the plain attention"
    pairs = [(b, hq) for b in range(len(lens)) for hq in range(hkv * group)]
    ref = _oracle(kq, vq, kp, vp, q, pairs, lens, slots_fn, group, scale, tau)
    got = sparse.cpu().numpy()
    for pr in pairs:
        assert_attention_close(got[pr][None], ref[pr][None])
    # the oracle drops a large share of the rows here, so the check is not vacuous
    b0, h0 = pairs[0]
    sl = np.asarray(slots_fn(b0, h0 // group, lens[b0]), dtype=np.int64)
    kc = oracle_cache(kq, *unpack(kq, kp, rows=sl))
    from oracle import estimate as oest
    qr, p = oest.prepare_query(q[b0, h0][None].double().numpy(), kq.D64, kq.S64)
    lg = scale * oest.scores(qr, p, kc.norm, kc.codes, kc.rnorm, kc.bits, kq.c)[0]
    w = np.exp(lg - lg.max())
    w /= w.sum()
    assert np.mean(w < tau) > 0.3
