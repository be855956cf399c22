"""GPU checks of the C-ABI boundary beyond the data paths' parity: search with large k
(32 < k <= 1024, the shared-memory top-k scan and merge) against the oracle's full sort, and the
bounded-wait failure path (a wait that runs out reports TQ_ETIMEOUT through tq_device_status and
leaves the context usable)."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oattn
from oracle import search as osearch
from parity import (Quantizer, assert_attention_close, assert_topk_equivalent, oracle_heads,
                    oracle_scores_from_packed, unpack)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_06_b200 import tq as _tq
    return _tq


def _enc(tq, q, x):
    packed = tq.Packed.allocate(q.ctx, x.shape[0])
    tq.encode_kv(q.ctx, x.cuda(), packed)
    torch.cuda.synchronize()
    return packed


@pytest.mark.parametrize("d,bits,m", [(128, 2, 128), (64, 1, 0), (1024, 3, 1024)])
def test_search_large_k(tq, d, bits, m):
    """k = 33 (just past the warp lists), 100, 257 and 1024 over 5003 rows (several shards, a
    ragged last block) with 9 queries (a ragged tile of 4)."""
    n, nq = 5003, 9
    q = Quantizer(d, bits, m, seed=140 + bits)
    X = synth.unit_rows(n, d, seed=141)
    Q = synth.unit_rows(nq, d, seed=142)
    packed = _enc(tq, q, X)
    codes, sbits, norm, rnorm = unpack(q, packed)
    ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
    for k in (33, 100, 257, 1024):
        s, i = tq.search_topk(q.ctx, Q.cuda(), packed, k)
        torch.cuda.synchronize()
        ref_s, _ = osearch.topk(ref_full, k)
        ss = s.cpu().numpy()
        assert np.all(ss[:, :-1] >= ss[:, 1:]), "lists are sorted best first"
        assert_topk_equivalent(ss, i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)


def test_search_large_k_edges(tq):
    """k = n (every row returned), fewer rows than one scan block, and duplicated rows (equal
    scores come back in index order)."""
    d, bits, m = 128, 2, 128
    q = Quantizer(d, bits, m, seed=150)
    Q = synth.unit_rows(5, d, seed=151)
    for n in (40, 129, 600):
        X = synth.unit_rows(n, d, seed=152 + n)
        packed = _enc(tq, q, X)
        codes, sbits, norm, rnorm = unpack(q, packed)
        ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
        k = min(n, 100) if n != 40 else 40
        s, i = tq.search_topk(q.ctx, Q.cuda(), packed, k)
        torch.cuda.synchronize()
        ref_s, _ = osearch.topk(ref_full, k)
        assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)
    X = synth.unit_rows(300, d, seed=160)
    packed = _enc(tq, q, torch.cat([X, X]))
    s, i = tq.search_topk(q.ctx, Q.cuda(), packed, 64)
    ii, ss = i.cpu().numpy(), s.cpu().numpy()
    for r in range(Q.shape[0]):
        assert np.array_equal(ii[r, 0::2] + 300, ii[r, 1::2])
        assert np.array_equal(ss[r, 0::2], ss[r, 1::2])


def _tensor_core_case(tq, seed):
    d, hkv, group, L = 128, 2, 4, 1504  # a context stride that is a multiple of 16 (value blocks)
    kq = Quantizer(d, 2, d, seed=seed)
    vq = Quantizer(d, 3, 0, seed=seed + 1, layout=1)
    K = synth.channel_scaled(1, hkv, L, d, seed=seed + 2)
    V = synth.channel_scaled(1, hkv, L, d, seed=seed + 3)
    kp = tq.Packed.allocate(kq.ctx, hkv * L)
    vp = tq.Packed.allocate(vq.ctx, hkv * L)
    tq.encode_kv(kq.ctx, K.reshape(-1, d).cuda(), kp)
    tq.encode_kv(vq.ctx, V.reshape(-1, d).cuda(), vp)
    q = synth.decode_queries(1, hkv * group, d, seed=seed + 4)
    lens = torch.tensor([L - 5], dtype=torch.int32)
    return kq, vq, kp, vp, q, lens, L, hkv, group


def test_bounded_wait_runs_out_and_reports_timeout(tq):
    """The test hook arms one barrier of every attention CTA for bytes that no copy sends: the
    bounded wait runs out, the kernel raises the device flag, drains the copies it had issued and
    returns; tq_device_status returns TQ_ETIMEOUT with the flag.  After clearing, the same call
    runs normally and matches the oracle: the context stayed usable."""
    kq, vq, kp, vp, q, lens, L, hkv, group = _tensor_core_case(tq, 170)
    assert tq.device_status(clear=True) == 0
    flags = ctypes.c_int32(-1)
    try:
        tq.debug_wait_probe(0, 256)
        out = tq.attend_decode(kq.ctx, vq.ctx, q.cuda(), kp, vp, lens.cuda(), L, n_kv_heads=hkv, ctx_stride=L)
        st = tq.LIB.tq_device_status(0, ctypes.byref(flags), 0)
        assert st == tq.TQ_ETIMEOUT, tq.LIB.tq_last_error()
        assert flags.value & tq.DEVFLAG_STAGING_TIMEOUT
        with pytest.raises(tq.TqError) as e:
            tq.check_device(0, clear=True)
        assert e.value.status == tq.TQ_ETIMEOUT and "gave up waiting" in str(e.value)
    finally:
        tq.debug_wait_probe(0, 0)
    assert tq.LIB.tq_device_status(0, ctypes.byref(flags), 0) == 0 and flags.value == 0
    out = tq.attend_decode(kq.ctx, vq.ctx, q.cuda(), kp, vp, lens.cuda(), L, n_kv_heads=hkv, ctx_stride=L)
    torch.cuda.synchronize()
    assert tq.device_status() == 0
    slots = lambda b, h, n: oattn.token_slots(b, h, n, hkv, ctx_stride=L)
    pairs = [(0, h) for h in range(hkv * group)]
    ref = oracle_heads(kq, vq, kp, vp, q, pairs, lens.numpy(), slots, group)
    got = out.cpu().numpy()
    for pr in pairs:
        assert_attention_close(got[pr][None], ref[pr][None])

