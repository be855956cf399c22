"""GPU parity of every C-ABI data call against the fp64 oracle, at sizes the oracle finishes in
seconds that still span several tiles / splits and a ragged tail.

Stage isolation: scores, attention and search are checked against the oracle evaluated on the
library's OWN packed bytes (decoded by the oracle's unpacker), so that an allowed near-threshold
code flip in encode cannot mask or fake an error downstream; encode itself is checked against
the oracle's encoding with the threshold band.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oattn
from oracle import encode as oenc
from oracle import search as osearch
from parity import (Quantizer, assert_attention_close, assert_scores_close, assert_topk_equivalent,
                    compare_encode, oracle_cache, oracle_scores_from_packed, unpack)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_06_b200 import tq as _tq
    return _tq


def _enc(tq, q, x, slots=None, capacity=None):
    cap = capacity if capacity is not None else x.shape[0]
    packed = tq.Packed.allocate(q.ctx, cap)
    tq.encode_kv(q.ctx, x.cuda(), packed, slots=None if slots is None else slots.cuda())
    torch.cuda.synchronize()
    return packed


@pytest.mark.parametrize("d", [8, 16, 32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_encode_all_dims_and_bits(tq, d, bits):
    m = min(d, 128) if d >= 32 else 32
    n = 1000 + 37
    q = Quantizer(d, bits, m, seed=d * 10 + bits)
    g = torch.Generator().manual_seed(d + bits)
    x = torch.randn(n, d, generator=g) * torch.exp(torch.randn(d, generator=g))
    packed = _enc(tq, q, x)
    codes, sbits, norm, rnorm = unpack(q, packed)
    compare_encode(q, q.oracle_encode(x.double().numpy()), codes, sbits, norm, rnorm)


@pytest.mark.parametrize("d,m,bits", [(128, 128, 2), (256, 128, 3), (1024, 1024, 1)])
def test_encode_large_batch_projection(tq, d, m, bits):
    """More rows than the fused small-batch encode takes: the separate QJL projection kernel
    (tensor cores, 3 x TF32) with a ragged last row tile."""
    n = 4096 + 300
    q = Quantizer(d, bits, m, seed=3 * d + bits)
    g = torch.Generator().manual_seed(d + m)
    x = torch.randn(n, d, generator=g) * torch.exp(torch.randn(d, generator=g))
    packed = _enc(tq, q, x)
    codes, sbits, norm, rnorm = unpack(q, packed)
    compare_encode(q, q.oracle_encode(x.double().numpy()), codes, sbits, norm, rnorm)


@pytest.mark.parametrize("m", [0, 32, 96])
def test_encode_mse_only_and_odd_m(tq, m):
    d, bits, n = 128, 3, 777
    q = Quantizer(d, bits, m, seed=5)
    x = torch.randn(n, d, generator=torch.Generator().manual_seed(1))
    packed = _enc(tq, q, x)
    codes, sbits, norm, rnorm = unpack(q, packed)
    compare_encode(q, q.oracle_encode(x.double().numpy()), codes, sbits, norm, rnorm)


def test_encode_bf16_strided_and_slots(tq):
    d, bits, m, n = 128, 2, 128, 333
    q = Quantizer(d, bits, m, seed=9)
    base = synth.channel_scaled(1, 1, n, d + 64, seed=3)[0, 0]       # bf16 [n, d+64]
    x = base[:, :d]                                                  # row stride d + 64
    cap = 1000
    slots = torch.randperm(cap, generator=torch.Generator().manual_seed(2))[:n].to(torch.int64)
    packed = tq.Packed.allocate(q.ctx, cap)
    tq.encode_kv(q.ctx, base.cuda()[:, :d], packed, slots=slots.cuda())
    torch.cuda.synchronize()
    codes, sbits, norm, rnorm = unpack(q, packed, rows=slots)
    compare_encode(q, q.oracle_encode(x.double().numpy()), codes, sbits, norm, rnorm)
    # untouched slots stay zero
    mask = torch.ones(cap, dtype=torch.bool)
    mask[slots] = False
    assert packed.codes.cpu()[mask].abs().sum() == 0


def test_encode_zero_vector_and_out_of_range_slots(tq):
    d, bits, m = 64, 2, 64
    q = Quantizer(d, bits, m, seed=1)
    x = torch.randn(4, d)
    x[1] = 0
    slots = torch.tensor([0, 1, 5, -1], dtype=torch.int64)   # 5 and -1 are outside capacity 4
    packed = tq.Packed.allocate(q.ctx, 4)
    packed.norm.fill_(-7.0)
    tq.encode_kv(q.ctx, x.cuda(), packed, slots=slots.cuda())
    torch.cuda.synchronize()
    nrm = packed.norm.cpu()
    assert nrm[1].item() == 0.0 and nrm[2].item() == -7.0 and nrm[3].item() == -7.0
    codes, sbits, norm, rnorm = unpack(q, packed, rows=[0, 1])
    compare_encode(q, q.oracle_encode(x[:2].double().numpy()), codes, sbits, norm, rnorm)


def test_tiny_config_scores(tq):
    """Tiny: one head, d=128, 4096 fp32 keys with outlier channels, 8 queries, 2 MSE bits +
    QJL m=128; exact and estimated logits."""
    keys, queries = synth.tiny(seed=0)
    q = Quantizer(128, 2, 128, seed=0)
    packed = _enc(tq, q, keys)
    codes, sbits, norm, rnorm = unpack(q, packed)
    stats = compare_encode(q, q.oracle_encode(keys.double().numpy()), codes, sbits, norm, rnorm)
    got = tq.scores(q.ctx, queries.cuda(), packed).cpu().numpy()
    ref = oracle_scores_from_packed(q, queries.double().numpy(), codes, sbits, norm, rnorm)
    assert_scores_close(got, ref)
    # end to end the library estimate is as close to the exact logits <q, k> as the oracle's own
    # encode + estimate (the estimator's noise, not the implementation, sets that distance)
    exact = queries.double().numpy() @ keys.double().numpy().T
    enc = q.oracle_encode(keys.double().numpy())
    own = oracle_scores_from_packed(q, queries.double().numpy(), enc.codes, enc.bits, enc.norm, enc.rnorm)
    rel_gpu = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    rel_oracle = np.linalg.norm(own - exact) / np.linalg.norm(exact)
    assert abs(rel_gpu - rel_oracle) < 0.02 * rel_oracle, (rel_gpu, rel_oracle)
    assert stats["code_flips"] <= 0.0001 * codes.size


def test_scores_bf16_queries_and_small_d(tq):
    for d, bits, m in [(8, 1, 32), (16, 4, 64), (256, 3, 256)]:
        q = Quantizer(d, bits, m, seed=d)
        x = torch.randn(501, d, generator=torch.Generator().manual_seed(d))
        qq = torch.randn(13, d, generator=torch.Generator().manual_seed(d + 1)).to(torch.bfloat16)
        packed = _enc(tq, q, x)
        codes, sbits, norm, rnorm = unpack(q, packed)
        got = tq.scores(q.ctx, qq.cuda(), packed).cpu().numpy()
        ref = oracle_scores_from_packed(q, qq.double().numpy(), codes, sbits, norm, rnorm)
        assert_scores_close(got, ref)


def _attention_case(tq, d, kbits, km, vbits, batch, hkv, group, lens, paged, qdtype, seed, vlayout=0, norm_bits=32):
    kq = Quantizer(d, kbits, km, seed=seed, norm_bits=norm_bits)
    vq = Quantizer(d, vbits, 0, seed=seed + 50, layout=vlayout, norm_bits=norm_bits)
    hq = hkv * group
    maxlen = int(max(lens))
    blk = synth.BLOCK_TOKENS
    lens_t = torch.tensor(lens, dtype=torch.int32)
    if paged:
        table, nblocks = synth.shuffled_block_table(lens_t, seed=seed + 7)
        cap = nblocks * hkv * blk
    else:
        table = None
        maxlen = (maxlen + 15) // 16 * 16 if vlayout == 1 else maxlen
        cap = batch * hkv * maxlen
    K = synth.channel_scaled(batch, hkv, maxlen, d, seed=seed + 1)
    V = synth.channel_scaled(batch, hkv, maxlen, d, seed=seed + 2)
    # slots of every (b, h, t < len)
    rows, slots = [], []
    for b in range(batch):
        for h in range(hkv):
            sl = oattn.token_slots(b, h, lens[b], hkv, ctx_stride=maxlen,
                                   block_table=None if table is None else table.numpy())
            rows.append((b, h, lens[b]))
            slots.append(sl)
    kx = torch.cat([K[b, h, :L] for b, h, L in rows])
    vx = torch.cat([V[b, h, :L] for b, h, L in rows])
    sl = torch.as_tensor(np.concatenate(slots), dtype=torch.int64)
    kp = tq.Packed.allocate(kq.ctx, cap)
    vp = tq.Packed.allocate(vq.ctx, cap)
    tq.encode_kv(kq.ctx, kx.cuda(), kp, slots=sl.cuda())
    tq.encode_kv(vq.ctx, vx.cuda(), vp, slots=sl.cuda())
    qx = synth.decode_queries(batch, hq, d, seed=seed + 3, dtype=qdtype)
    out = tq.attend_decode(kq.ctx, vq.ctx, qx.cuda(), kp, vp, lens_t.cuda(), int(max(lens)), n_kv_heads=hkv,
                           ctx_stride=maxlen, block_table=None if table is None else table.cuda(),
                           block_size=blk)
    torch.cuda.synchronize()
    kc = oracle_cache(kq, *unpack(kq, kp))
    vc = oracle_cache(vq, *unpack(vq, vp))
    ref = oattn.attend_decode(qx.double().numpy(), kc, vc, lens, hkv, kq.D64, kq.S64, kq.c, vq.D64, vq.c,
                              ctx_stride=maxlen, block_table=None if table is None else table.numpy())
    assert_attention_close(out.cpu().numpy(), ref)
    assert tq.device_status() == 0
    # encode parity on these rows too
    compare_encode(kq, kq.oracle_encode(kx.double().numpy()), *unpack(kq, kp, rows=sl))
    return out


@pytest.mark.parametrize("kbits,vbits", [(2, 3), (3, 2)])
def test_attention_contiguous_gqa4(tq, kbits, vbits):
    _attention_case(tq, 128, kbits, 128, vbits, batch=2, hkv=2, group=4, lens=[1500, 333], paged=False,
                    qdtype=torch.bfloat16, seed=11 + kbits)


def test_attention_paged_ragged(tq):
    _attention_case(tq, 128, 2, 128, 3, batch=3, hkv=2, group=4, lens=[700, 16, 1031], paged=True,
                    qdtype=torch.bfloat16, seed=21)


@pytest.mark.parametrize("group", [1, 2, 8])
def test_attention_group_sizes_and_dims(tq, group):
    _attention_case(tq, 64, 2, 64, 2, batch=1, hkv=2, group=group, lens=[300], paged=False,
                    qdtype=torch.float32, seed=31 + group)


def test_attention_d256_and_multi_split(tq):
    _attention_case(tq, 256, 3, 256, 3, batch=1, hkv=1, group=4, lens=[5000], paged=False,
                    qdtype=torch.float32, seed=41)


def test_attention_empty_and_single_token(tq):
    out = _attention_case(tq, 128, 2, 128, 3, batch=3, hkv=1, group=4, lens=[0, 1, 17], paged=True,
                          qdtype=torch.float32, seed=51)
    assert torch.all(out[0] == 0)


@pytest.mark.parametrize("d,bits,m", [(128, 2, 128), (256, 1, 256), (1024, 3, 1024)])
def test_search_topk_small(tq, d, bits, m):
    n, nq, k = 5003, 17, 10
    q = Quantizer(d, bits, m, seed=61 + bits)
    X = synth.unit_rows(n, d, seed=0)
    Q = synth.unit_rows(nq, d, seed=1)
    packed = _enc(tq, q, X)
    codes, sbits, norm, rnorm = unpack(q, packed)
    s, i = tq.search_topk(q.ctx, Q.cuda(), packed, k)
    torch.cuda.synchronize()
    ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
    ref_s, ref_i = osearch.topk(ref_full, k)
    assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)


def test_search_k_edge_cases(tq):
    d, bits, m = 64, 2, 64
    q = Quantizer(d, bits, m, seed=3)
    X = synth.unit_rows(40, d, seed=4)
    Q = synth.unit_rows(3, d, seed=5)
    packed = _enc(tq, q, X)
    codes, sbits, norm, rnorm = unpack(q, packed)
    ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
    for k in (1, 32):
        s, i = tq.search_topk(q.ctx, Q.cuda(), packed, k)
        ref_s, _ = osearch.topk(ref_full, k)
        assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)
    # duplicate rows: equal scores must come back in index order
    Xd = torch.cat([X[:5], X[:5]])
    pd = _enc(tq, q, Xd)
    s, i = tq.search_topk(q.ctx, Q.cuda(), pd, 10)
    ii, ss = i.cpu().numpy(), s.cpu().numpy()
    for r in range(3):
        assert sorted(ii[r].tolist()) == list(range(10))
        for a in range(9):
            assert ss[r, a] >= ss[r, a + 1]
            if ss[r, a] == ss[r, a + 1]:
                assert ii[r, a] < ii[r, a + 1]


@pytest.mark.parametrize("d,bits", [(128, 1), (128, 3), (512, 2)])
def test_search_tensor_core_scan_edges(tq, d, bits):
    """Bit-plane tensor-core scan (d in 128..1024, m = d, 1..3 bits): databases shorter than one
    128-row block, ragged tails that are not a multiple of 4 rows, k = n, k = 32, query counts
    that leave a partial tile of 8, duplicate rows (equal scores in index order), and a norm array
    at a 4-byte offset (which takes the CUDA-core scan)."""
    q = Quantizer(d, bits, d, seed=70 + bits)
    Q = synth.unit_rows(11, d, seed=71)
    for n, k in ((1, 1), (3, 3), (40, 32), (129, 10), (1030, 32)):
        X = synth.unit_rows(n, d, seed=72 + n)
        packed = _enc(tq, q, X)
        codes, sbits, norm, rnorm = unpack(q, packed)
        ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
        ref_s, _ = osearch.topk(ref_full, k)
        s, i = tq.search_topk(q.ctx, Q.cuda(), packed, k)
        torch.cuda.synchronize()
        assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)
    X = synth.unit_rows(300, d, seed=73)
    Xd = torch.cat([X, X])
    pd = _enc(tq, q, Xd)
    s, i = tq.search_topk(q.ctx, Q.cuda(), pd, 32)
    ii, ss = i.cpu().numpy(), s.cpu().numpy()
    for r in range(Q.shape[0]):
        for a in range(31):
            assert ss[r, a] >= ss[r, a + 1]
            if ss[r, a] == ss[r, a + 1]:
                assert ii[r, a] < ii[r, a + 1]
        # row j and its copy j + 300 score the same, so the list holds the pairs (j, j + 300)
        assert np.array_equal(ii[r, 0::2] + 300, ii[r, 1::2])
        assert np.array_equal(ss[r, 0::2], ss[r, 1::2])
    # a norm array one float off a 16-byte boundary: same results through the CUDA-core scan
    X = synth.unit_rows(1000, d, seed=74)
    packed = _enc(tq, q, X)
    base_s, base_i = tq.search_topk(q.ctx, Q.cuda(), packed, 10)
    nbuf = torch.empty(1001, dtype=torch.float32, device="cuda")
    rbuf = torch.empty(1001, dtype=torch.float32, device="cuda")
    nbuf[1:].copy_(packed.norm)
    rbuf[1:].copy_(packed.rnorm)
    shifted = tq.Packed(packed.codes, nbuf[1:], packed.signs, rbuf[1:])
    s2, i2 = tq.search_topk(q.ctx, Q.cuda(), shifted, 10)
    torch.cuda.synchronize()
    codes, sbits, norm, rnorm = unpack(q, packed)
    ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
    ref_s, _ = osearch.topk(ref_full, 10)
    for got_s, got_i in ((base_s, base_i), (s2, i2)):
        assert_topk_equivalent(got_s.cpu().numpy(), got_i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)


@pytest.mark.parametrize("d,bits", [(128, 2), (256, 1), (512, 3), (1024, 1), (1024, 3)])
def test_search_tcgen05_scan(tq, d, bits):
    """tcgen05 scan (at least 32 queries, k <= 16, d in 128..1024, m = d): a ragged second tile of
    64 queries, databases shorter than one 128-row block and with ragged tails, k = 1, 10, 16,
    and duplicate rows (equal scores in index order)."""
    q = Quantizer(d, bits, d, seed=80 + bits)
    Q = synth.unit_rows(70, d, seed=81)
    for n, k in ((1, 1), (3, 3), (129, 10), (1030, 16), (5003, 10)):
        X = synth.unit_rows(n, d, seed=82 + n)
        packed = _enc(tq, q, X)
        codes, sbits, norm, rnorm = unpack(q, packed)
        ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
        ref_s, _ = osearch.topk(ref_full, k)
        s, i = tq.search_topk(q.ctx, Q.cuda(), packed, k)
        torch.cuda.synchronize()
        assert tq.device_status() == 0
        assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)
    X = synth.unit_rows(300, d, seed=83)
    pd = _enc(tq, q, torch.cat([X, X]))
    s, i = tq.search_topk(q.ctx, Q.cuda(), pd, 16)
    ii, ss = i.cpu().numpy(), s.cpu().numpy()
    for r in range(Q.shape[0]):
        assert np.all(ss[r, :-1] >= ss[r, 1:])
        # row j and its copy j + 300 score the same, so the list holds the pairs (j, j + 300)
        assert np.array_equal(ii[r, 0::2] + 300, ii[r, 1::2])
        assert np.array_equal(ss[r, 0::2], ss[r, 1::2])


def test_search_tcgen05_bf16_queries_many_shards(tq):
    """bf16 queries through the tcgen05 scan, with a database long enough for one shard per SM
    (two 64-query tiles x 67 shards of 7 row blocks) and k = 16."""
    d, bits, n, nq, k = 256, 2, 60000, 100, 16
    q = Quantizer(d, bits, d, seed=95)
    X = synth.unit_rows(n, d, seed=96)
    Q = synth.unit_rows(nq, d, seed=97).to(torch.bfloat16)
    packed = _enc(tq, q, X)
    codes, sbits, norm, rnorm = unpack(q, packed)
    ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
    ref_s, _ = osearch.topk(ref_full, k)
    s, i = tq.search_topk(q.ctx, Q.cuda(), packed, k)
    torch.cuda.synchronize()
    assert tq.device_status() == 0
    assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)


@pytest.mark.parametrize("d,bits", [(8, 1), (64, 2), (128, 3), (128, 4), (256, 2)])
def test_encode_block16_layout(tq, d, bits):
    """Values in the token-transposed 16-slot block layout, written at scattered slots (several
    vectors share each block word, so concurrent writers must not clobber each other)."""
    n, cap = 300, 512
    q = Quantizer(d, bits, 0, seed=d + 7 * bits, layout=1)
    x = torch.randn(n, d, generator=torch.Generator().manual_seed(d)) * 3
    slots = torch.randperm(cap, generator=torch.Generator().manual_seed(bits))[:n].to(torch.int64)
    packed = tq.Packed.allocate(q.ctx, cap)
    packed.codes.fill_(0xA5)                        # stale bits must be cleared for written slots
    tq.encode_kv(q.ctx, x.cuda(), packed, slots=slots.cuda())
    torch.cuda.synchronize()
    codes, sbits, norm, rnorm = unpack(q, packed, rows=slots)
    compare_encode(q, q.oracle_encode(x.double().numpy()), codes, sbits, norm, rnorm)


@pytest.mark.parametrize("layout,bits", [(0, 1), (0, 2), (0, 3), (0, 4), (1, 2), (1, 3), (1, 4), (1, 1)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_encode_bulk_rows_d128(tq, layout, bits, dtype):
    """More rows than the fused small-batch limit at d = 128 (one row per thread): row layout
    and the token-block layout (whole blocks by ballots, a ragged tail of 13 rows through the
    general kernel next to it, stale bytes in the untouched slots of the last block)."""
    n = 5011
    cap = (n + 15) // 16 * 16 + 32
    q = Quantizer(128, bits, 0, seed=600 + 10 * bits + layout, layout=layout)
    x = (torch.randn(n, 128, generator=torch.Generator().manual_seed(bits)) *
         torch.exp(torch.randn(128, generator=torch.Generator().manual_seed(7)))).to(dtype)
    x[17] = 0  # a zero vector
    packed = tq.Packed.allocate(q.ctx, cap)
    packed.codes.fill_(0x5A)
    tq.encode_kv(q.ctx, x.cuda(), packed)
    torch.cuda.synchronize()
    rows = np.arange(n)
    codes, sbits, norm, rnorm = unpack(q, packed, rows=rows)
    compare_encode(q, q.oracle_encode(x.double().numpy()), codes, sbits, norm, rnorm)
    if layout == 1:
        # slots past n in the last partial block keep their earlier bytes (the tail kernel only
        # changes the bits of the slots it writes)
        tail = np.arange(n, (n + 15) // 16 * 16)
        stale = unpack(q, packed, rows=tail)[0]
        full = oenc.unpack_codes_block16(np.full((16, packed.codes.shape[1]), 0x5A, dtype=np.uint8), 128, bits)
        assert np.array_equal(stale, full[tail % 16])


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_encode_bulk_keys_qjl_bf16(tq, bits):
    """bf16 keys with a dense JL matrix (d = m = 128) past the fused small-batch limit: the
    tensor-core encode (rotation as a bf16 MMA, z = S r as three TF32 products), with scattered
    slots, a zero vector, a ragged last tile and out-of-range slots that must be skipped."""
    n, d = 5011, 128
    cap = n + 64
    q = Quantizer(d, bits, 128, seed=700 + bits)
    x = (torch.randn(n, d, generator=torch.Generator().manual_seed(40 + bits)) *
         torch.exp(torch.randn(d, generator=torch.Generator().manual_seed(8)))).to(torch.bfloat16)
    x[5] = 0
    slots = torch.randperm(cap, generator=torch.Generator().manual_seed(bits))[:n].to(torch.int64)
    slots[9] = cap + 3  # out of range: not written
    packed = tq.Packed.allocate(q.ctx, cap)
    packed.codes.fill_(0xA5)
    tq.encode_kv(q.ctx, x.cuda(), packed, slots=slots.cuda())
    torch.cuda.synchronize()
    keep = np.array([i for i in range(n) if i != 9])
    codes, sbits, norm, rnorm = unpack(q, packed, rows=slots.numpy()[keep])
    compare_encode(q, q.oracle_encode(x.double().numpy()[keep]), codes, sbits, norm, rnorm)


@pytest.mark.parametrize("vbits", [2, 3])
def test_attention_block16_values_contiguous(tq, vbits):
    _attention_case(tq, 128, 2, 128, vbits, batch=2, hkv=2, group=4, lens=[1500, 333], paged=False,
                    qdtype=torch.bfloat16, seed=81 + vbits, vlayout=1)


def test_attention_block16_values_paged(tq):
    _attention_case(tq, 128, 3, 128, 3, batch=3, hkv=2, group=4, lens=[700, 16, 1031], paged=True,
                    qdtype=torch.bfloat16, seed=91, vlayout=1)


@pytest.mark.parametrize("kbits,km,vbits", [(1, 128, 2), (2, 128, 3), (3, 128, 3), (2, 0, 2), (3, 0, 3)])
def test_attention_tensor_core_path_variants(tq, kbits, km, vbits):
    """d = 128, 4 query heads per KV head, token-block values: the tensor-core path
    (attend_mma.cu); ragged lengths, several 256-token chunks, a sequence shorter than one
    block."""
    _attention_case(tq, 128, kbits, km, vbits, batch=3, hkv=2, group=4, lens=[2600, 5, 777], paged=False,
                    qdtype=torch.bfloat16, seed=101 + 10 * kbits + vbits, vlayout=1)


def test_attention_tensor_core_path_paged_and_empty(tq):
    out = _attention_case(tq, 128, 2, 128, 3, batch=4, hkv=3, group=4, lens=[0, 1, 1500, 33], paged=True,
                          qdtype=torch.float32, seed=131, vlayout=1)
    assert torch.all(out[0] == 0)


def test_attention_tensor_core_path_matches_general_kernel(tq):
    """Same packed K and V (bits identical), read once by the general CUDA-core kernel (row-major
    values) and once by the tensor-core kernel (token-block values)."""
    d, hkv, group, lens = 128, 2, 4, [3000, 1200]
    kq = Quantizer(d, 2, d, seed=141)
    v_rows = Quantizer(d, 3, 0, seed=142, layout=0)
    v_blk = Quantizer(d, 3, 0, seed=142, layout=1)
    maxlen = 3008
    K = synth.channel_scaled(2, hkv, maxlen, d, seed=143).reshape(-1, d)
    V = synth.channel_scaled(2, hkv, maxlen, d, seed=144).reshape(-1, d)
    kp = tq.Packed.allocate(kq.ctx, K.shape[0])
    vr = tq.Packed.allocate(v_rows.ctx, V.shape[0])
    vb = tq.Packed.allocate(v_blk.ctx, V.shape[0])
    tq.encode_kv(kq.ctx, K.cuda(), kp)
    tq.encode_kv(v_rows.ctx, V.cuda(), vr)
    tq.encode_kv(v_blk.ctx, V.cuda(), vb)
    q = synth.decode_queries(2, hkv * group, d, seed=145).cuda()
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    o_gen = tq.attend_decode(kq.ctx, v_rows.ctx, q, kp, vr, lens_t, maxlen, n_kv_heads=hkv, ctx_stride=maxlen)
    o_tc = tq.attend_decode(kq.ctx, v_blk.ctx, q, kp, vb, lens_t, maxlen, n_kv_heads=hkv, ctx_stride=maxlen)
    torch.cuda.synchronize()
    assert_attention_close(o_tc.cpu().numpy(), o_gen.cpu().numpy())


# ------------------------------------------------------------------ fp16 norms (tq_spec.norm_bits = 16)
@pytest.mark.parametrize("path", ["bulk_keys_bf16", "bulk_values_block_bf16", "bulk_fp32", "small_batch", "srht"])
def test_norm16_encode_paths(tq, path):
    """Norms stored in fp16 through every encode path: the stored norm is the oracle's fp16 norm
    (within one half ulp, the library rounding its fp32 norm), codes and signs as with fp32 norms."""
    d = 128
    n = {"small_batch": 333}.get(path, 5011)
    layout = 1 if path == "bulk_values_block_bf16" else 0
    m = 0 if path == "bulk_values_block_bf16" else 128
    q = Quantizer(d, 2, m, seed=800 + len(path), layout=layout, norm_bits=16, srht=(path == "srht"))
    x = (torch.randn(n, d, generator=torch.Generator().manual_seed(5)) *
         torch.exp(torch.randn(d, generator=torch.Generator().manual_seed(6))))
    if path != "bulk_fp32" and path != "small_batch":
        x = x.to(torch.bfloat16)
    x[3] = 0
    cap = (n + 15) // 16 * 16
    packed = tq.Packed.allocate(q.ctx, cap)
    assert packed.norm.dtype == torch.float16
    tq.encode_kv(q.ctx, x.cuda(), packed)
    torch.cuda.synchronize()
    rows = np.arange(n)
    compare_encode(q, q.oracle_encode(x.double().numpy()), *unpack(q, packed, rows=rows))


@pytest.mark.parametrize("vlayout", [0, 1])
def test_norm16_attention(tq, vlayout):
    """fp16 norms through the general (row values) and the tensor-core (token-block values)
    attention paths, paged and ragged; the oracle reads the library's own stored norms."""
    _attention_case(tq, 128, 2, 128, 3, batch=3, hkv=2, group=4, lens=[700, 16, 1031], paged=True,
                    qdtype=torch.bfloat16, seed=97, vlayout=vlayout, norm_bits=16)


def test_norm16_scores_and_search(tq):
    """fp16 norms in tq_scores and the three search scans (CUDA cores for few queries, tcgen05 for
    many, the large-k scan)."""
    d, n = 128, 3001
    q = Quantizer(d, 2, d, seed=99, norm_bits=16)
    X = synth.unit_rows(n, d, seed=7) * 3.0
    packed = _enc(tq, q, X)
    codes, sbits, norm, rnorm = unpack(q, packed)
    for nq, k in ((5, 10), (40, 10), (6, 100)):
        Q = synth.unit_rows(nq, d, seed=8 + nq)
        ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
        if nq == 5:
            assert_scores_close(tq.scores(q.ctx, Q.cuda(), packed).cpu().numpy(), ref_full)
        s, i = tq.search_topk(q.ctx, Q.cuda(), packed, k)
        ref_s, _ = osearch.topk(ref_full, k)
        assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)
    assert tq.device_status() == 0
