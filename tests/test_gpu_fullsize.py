"""GPU parity at the workloads' full sizes, checked on sampled outputs that the oracle computes one
by one (stage-isolated: the oracle reads the library's own packed bytes):

  * Llama-3.1-8B-shaped decode layer: batch 1, 32 q / 8 KV heads, d 128, context 32768, K at 3
    and 4 bits (b-1 MSE bits + QJL m=128), V 3 bits; every query head checked;
  * long context: batch 4, 8 KV heads (32 q), context 131072, K 4 bits, V 2 bits; encode the
    whole cache, then 64 decode steps that append and encode one token per head and attend over
    the full cache; sampled heads checked after the last step;
  * vector search: 10^6 unit vectors d 1024, queries likewise, 2 and 4 bits per coordinate
    (QJL m 1024), top-10; sampled queries checked against the oracle's full scan; recall@10
    against exact fp64 search printed;
  * ragged paged serving: batch 64, lengths U[1024, 32768], 16-token blocks in a shuffled table,
    K 3 bits, V 3 bits; sampled sequences (shortest, longest, random) checked.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oattn
from oracle import encode as oenc
from oracle import estimate as oest
from oracle import search as osearch
from parity import Quantizer, assert_attention_close, assert_topk_equivalent, compare_encode, oracle_heads, unpack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_06_b200 import tq as _tq
    return _tq


def _encode_heads(tq, q, X, ctx_stride, slots_of):
    """Encode [B, H, L, d] rows into a contiguous-slot cache."""
    B, H, L, d = X.shape
    cap = B * H * ctx_stride
    p = tq.Packed.allocate(q.ctx, cap)
    for b in range(B):
        for h in range(H):
            sl = torch.as_tensor(slots_of(b, h, L), dtype=torch.int64).cuda()
            tq.encode_kv(q.ctx, X[b, h].cuda(), p, slots=sl)
    torch.cuda.synchronize()
    return p


def _check_sampled_encode(q, packed, X2d, slots, n=2048, seed=0):
    rng = np.random.default_rng(seed)
    pick = rng.choice(len(slots), size=min(n, len(slots)), replace=False)
    rows = np.asarray(slots)[pick]
    compare_encode(q, q.oracle_encode(X2d[pick].double().numpy()), *unpack(q, packed, rows=rows))


@pytest.mark.parametrize("kbits", [3, 4])
def test_llama8b_decode_layer_full(tq, kbits):
    d, B, hkv, hq, ctx = 128, 1, 8, 32, 32768
    kq = Quantizer(d, kbits - 1, d, seed=500 + kbits)
    vq = Quantizer(d, 3, 0, seed=600, layout=1)
    K = synth.channel_scaled(B, hkv, ctx, d, seed=501)
    V = synth.channel_scaled(B, hkv, ctx, d, seed=502)
    slots_of = lambda b, h, L: oattn.token_slots(b, h, L, hkv, ctx_stride=ctx)
    kp = _encode_heads(tq, kq, K, ctx, slots_of)
    vp = _encode_heads(tq, vq, V, ctx, slots_of)
    q = synth.decode_queries(B, hq, d, seed=503)
    lens = torch.full((B,), ctx, dtype=torch.int32)
    out = tq.attend_decode(kq.ctx, vq.ctx, q.cuda(), kp, vp, lens.cuda(), ctx, n_kv_heads=hkv, ctx_stride=ctx)
    torch.cuda.synchronize()
    pairs = [(0, hh) for hh in range(hq)]
    ref = oracle_heads(kq, vq, kp, vp, q, pairs, lens, slots_of, hq // hkv)
    got = out.cpu().numpy()
    for pr in pairs:
        assert_attention_close(got[pr][None], ref[pr][None])
    all_slots = np.arange(B * hkv * ctx)
    _check_sampled_encode(kq, kp, K.reshape(-1, d), all_slots)
    _check_sampled_encode(vq, vp, V.reshape(-1, d), all_slots, seed=1)


def test_long_context_prefill_then_64_steps(tq):
    d, B, hkv, hq, ctx, steps = 128, 4, 8, 32, 131072, 64
    stride = ctx + steps
    kq = Quantizer(d, 3, d, seed=700)          # 4 bits = 3 MSE + 1 QJL
    vq = Quantizer(d, 2, 0, seed=701, layout=1)
    K = synth.channel_scaled(B, hkv, ctx, d, seed=702)
    V = synth.channel_scaled(B, hkv, ctx, d, seed=703)
    slots_of = lambda b, h, L: oattn.token_slots(b, h, L, hkv, ctx_stride=stride)
    kp = _encode_heads(tq, kq, K, stride, slots_of)
    vp = _encode_heads(tq, vq, V, stride, slots_of)
    newK = synth.channel_scaled(B, hkv, steps, d, seed=704)
    newV = synth.channel_scaled(B, hkv, steps, d, seed=705)
    lens = torch.full((B,), ctx, dtype=torch.int32).cuda()
    out = None
    for t in range(steps):
        sl = torch.as_tensor([(b * hkv + h) * stride + ctx + t for b in range(B) for h in range(hkv)],
                             dtype=torch.int64).cuda()
        tq.encode_kv(kq.ctx, newK[:, :, t].reshape(-1, d).cuda(), kp, slots=sl)
        tq.encode_kv(vq.ctx, newV[:, :, t].reshape(-1, d).cuda(), vp, slots=sl)
        lens += 1
        q = synth.decode_queries(B, hq, d, seed=800 + t).cuda()
        out = tq.attend_decode(kq.ctx, vq.ctx, q, kp, vp, lens, stride, n_kv_heads=hkv, ctx_stride=stride)
    torch.cuda.synchronize()
    pairs = [(0, 0), (1, 13), (2, 22), (3, 31)]
    ref = oracle_heads(kq, vq, kp, vp, q, pairs, [stride] * B, slots_of, hq // hkv)
    got = out.cpu().numpy()
    for pr in pairs:
        assert_attention_close(got[pr][None], ref[pr][None])
    # the appended tokens were encoded like every other row
    last = np.array([(b * hkv + h) * stride + ctx + steps - 1 for b in range(B) for h in range(hkv)])
    compare_encode(kq, kq.oracle_encode(newK[:, :, -1].reshape(-1, d).double().numpy()), *unpack(kq, kp, rows=last))


@pytest.mark.parametrize("bits", [2, 4])
def test_vector_search_million_rows(tq, bits):
    d, n, nq, k = 1024, 1_000_000, 1000, 10
    q = Quantizer(d, bits - 1, d, seed=900 + bits)
    X = synth.unit_rows(n, d, seed=0)
    Q = synth.unit_rows(nq, d, seed=1)
    db = tq.Packed.allocate(q.ctx, n)
    Xg = X.cuda()
    tq.encode_kv(q.ctx, Xg, db)
    del Xg
    s, i = tq.search_topk(q.ctx, Q.cuda(), db, k)
    torch.cuda.synchronize()
    s, i = s.cpu().numpy(), i.cpu().numpy()
    # sampled queries: the oracle's own full scan over the library's packed bytes
    sample = [0, 1, 17, 500, 999]
    qr, p = oest.prepare_query(Q[sample].double().numpy(), q.D64, q.S64)
    ref_s = np.full((len(sample), k), -np.inf)
    ref_i = np.zeros((len(sample), k), dtype=np.int64)
    step = 1 << 15
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        codes = oenc.unpack_codes(db.codes[r0:r1].cpu().numpy(), d, q.bits)
        sbits = oenc.unpack_signs(db.signs[r0:r1].cpu().numpy(), d)
        sc = oest.scores(qr, p, db.norm[r0:r1].double().cpu().numpy(), codes, db.rnorm[r0:r1].double().cpu().numpy(),
                         sbits, q.c)
        v, ix = osearch.topk(sc, k)
        cv = np.concatenate([ref_s, v], axis=1)
        ci = np.concatenate([ref_i, ix + r0], axis=1)
        for row in range(len(sample)):
            order = np.lexsort((ci[row], -cv[row]))[:k]
            ref_s[row], ref_i[row] = cv[row, order], ci[row, order]

    def oracle_scores_at(row, idx):
        codes = oenc.unpack_codes(db.codes[torch.as_tensor(idx)].cpu().numpy(), d, q.bits)
        sb = oenc.unpack_signs(db.signs[torch.as_tensor(idx)].cpu().numpy(), d)
        return oest.scores(qr[row:row + 1], p[row:row + 1], db.norm[torch.as_tensor(idx)].double().cpu().numpy(),
                           codes, db.rnorm[torch.as_tensor(idx)].double().cpu().numpy(), sb, q.c)[0]

    assert_topk_equivalent(s[sample], i[sample], oracle_scores_at, ref_s)
    # encode parity on sampled rows, recall@10 against exact fp64 search (reported)
    rows = np.random.default_rng(3).choice(n, size=2000, replace=False)
    compare_encode(q, q.oracle_encode(X[rows].double().numpy()), *unpack(q, db, rows=rows))
    _, exact = osearch.exact_topk(Q[sample].double().numpy(), X.numpy(), k, chunk=1 << 17)
    print(f"recall@10 ({bits} bits/coord, sampled queries): {osearch.recall_at_k(i[sample], exact):.3f}")


def test_ragged_paged_serving_step(tq):
    d, B, hkv, hq, blk = 128, 64, 8, 32, synth.BLOCK_TOKENS
    kq = Quantizer(d, 2, d, seed=1100)
    vq = Quantizer(d, 3, 0, seed=1101, layout=1)
    lens = synth.ragged_lengths(B, 1024, 32768, seed=1102)
    table, nblocks = synth.shuffled_block_table(lens, seed=1103)
    cap = nblocks * hkv * blk
    kp, vp = tq.Packed.allocate(kq.ctx, cap), tq.Packed.allocate(vq.ctx, cap)
    keep = {}
    for b in range(B):
        L = int(lens[b])
        Kb = synth.channel_scaled(1, hkv, L, d, seed=2000 + b)[0]
        Vb = synth.channel_scaled(1, hkv, L, d, seed=3000 + b)[0]
        for h in range(hkv):
            sl = oattn.token_slots(b, h, L, hkv, block_table=table.numpy())
            slt = torch.as_tensor(sl, dtype=torch.int64).cuda()
            tq.encode_kv(kq.ctx, Kb[h].cuda(), kp, slots=slt)
            tq.encode_kv(vq.ctx, Vb[h].cuda(), vp, slots=slt)
            if b in (0, 5) and h == 1:
                keep[b] = (Kb[h], sl)
    q = synth.decode_queries(B, hq, d, seed=1104)
    maxlen = int(lens.max())
    out = tq.attend_decode(kq.ctx, vq.ctx, q.cuda(), kp, vp, lens.cuda(), maxlen, n_kv_heads=hkv,
                           block_table=table.cuda(), block_size=blk)
    torch.cuda.synchronize()
    b_short, b_long = int(torch.argmin(lens)), int(torch.argmax(lens))
    pairs = [(b_short, 0), (b_short, 31), (b_long, 5), (b_long, 30), (7, 9), (40, 17)]
    paged_slots = lambda b, h, L: oattn.token_slots(b, h, L, hkv, block_table=table.numpy())
    ref = oracle_heads(kq, vq, kp, vp, q, pairs, lens.numpy(), paged_slots, hq // hkv)
    got = out.cpu().numpy()
    for pr in pairs:
        assert_attention_close(got[pr][None], ref[pr][None])
    for b, (Kh, sl) in keep.items():
        compare_encode(kq, kq.oracle_encode(Kh.double().numpy()), *unpack(kq, kp, rows=sl))
