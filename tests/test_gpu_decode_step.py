"""GPU parity of tq_decode_step (append the new K/V token of every (sequence, KV head), then
attend): the packed bytes it writes and the attention it returns must equal those of the
separate calls (tq_encode_kv for K, for V, then tq_attend_decode) on the same inputs, and the
attention must match the oracle evaluated on the library's own packed bytes; the appended rows
are checked against the oracle's encoding.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oattn
from parity import Quantizer, assert_attention_close, compare_encode, oracle_heads, unpack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_06_b200 import tq as _tq
    return _tq


def _clone(tq, ctx, p):
    c = tq.Packed.allocate(ctx, p.codes.shape[0])
    for name in ("codes", "signs", "norm", "rnorm"):
        a, b = getattr(p, name), getattr(c, name)
        if a is not None and a.numel():
            b.copy_(a)
    return c


def _packed_equal(a, b):
    for name in ("codes", "signs", "norm", "rnorm"):
        x, y = getattr(a, name), getattr(b, name)
        if x is not None and x.numel():
            assert torch.equal(x, y), name


def _step_case(tq, d, kbits, km, vbits, vlayout, batch, hkv, group, lens, paged, seed, kvdtype=torch.float32,
               qdtype=torch.bfloat16, srht=False, norm_bits=32):
    kq = Quantizer(d, kbits, km, seed=seed, srht=srht, norm_bits=norm_bits)
    vq = Quantizer(d, vbits, 0, seed=seed + 50, layout=vlayout, norm_bits=norm_bits)
    hq = hkv * group
    blk = synth.BLOCK_TOKENS
    new_lens = [L + 1 for L in lens]
    lens_new_t = torch.tensor(new_lens, dtype=torch.int32)
    if paged:
        table, nblocks = synth.shuffled_block_table(lens_new_t, seed=seed + 7)
        tab = table.numpy()
        cap = nblocks * hkv * blk
        stride = 0
    else:
        table, tab = None, None
        stride = (max(new_lens) + 15) // 16 * 16
        cap = batch * hkv * stride
    K = synth.channel_scaled(batch, hkv, max(new_lens), d, seed=seed + 1)
    V = synth.channel_scaled(batch, hkv, max(new_lens), d, seed=seed + 2)
    slots_of = lambda b, h, L: oattn.token_slots(b, h, L, hkv, ctx_stride=stride, block_table=tab)
    kp = tq.Packed.allocate(kq.ctx, cap)
    vp = tq.Packed.allocate(vq.ctx, cap)
    for b in range(batch):
        for h in range(hkv):
            if lens[b] == 0:
                continue
            sl = torch.as_tensor(slots_of(b, h, lens[b]), dtype=torch.int64).cuda()
            tq.encode_kv(kq.ctx, K[b, h, :lens[b]].cuda(), kp, slots=sl)
            tq.encode_kv(vq.ctx, V[b, h, :lens[b]].cuda(), vp, slots=sl)
    # the new token of every (b, h) sits at position lens[b]
    new_slots = np.array([slots_of(b, h, new_lens[b])[-1] for b in range(batch) for h in range(hkv)])
    knew = torch.stack([K[b, h, lens[b]] for b in range(batch) for h in range(hkv)]).to(kvdtype)
    vnew = torch.stack([V[b, h, lens[b]] for b in range(batch) for h in range(hkv)]).to(kvdtype)
    q = synth.decode_queries(batch, hq, d, seed=seed + 3, dtype=qdtype).cuda()
    kp2, vp2 = _clone(tq, kq.ctx, kp), _clone(tq, vq.ctx, vp)
    maxlen = max(new_lens)
    desc_args = dict(n_kv_heads=hkv, ctx_stride=stride, block_table=None if table is None else table.cuda(),
                     block_size=blk)
    lens_g = lens_new_t.cuda()
    sl_g = torch.as_tensor(new_slots, dtype=torch.int64).cuda()
    desc = tq.make_attn_desc(kq.ctx, vq.ctx, q.shape, kp, vp, lens_g, maxlen, **desc_args)
    out = tq.decode_step(kq.ctx, vq.ctx, q, knew.cuda(), vnew.cuda(), sl_g, desc)
    # the separate calls
    tq.encode_kv(kq.ctx, knew.cuda(), kp2, slots=sl_g)
    tq.encode_kv(vq.ctx, vnew.cuda(), vp2, slots=sl_g)
    out2 = tq.attend_decode(kq.ctx, vq.ctx, q, kp2, vp2, lens_g, maxlen, **desc_args)
    torch.cuda.synchronize()
    _packed_equal(kp, kp2)
    _packed_equal(vp, vp2)
    assert torch.equal(out, out2)
    assert tq.device_status() == 0
    pairs = [(b, h) for b in range(batch) for h in range(hq)]
    ref = oracle_heads(kq, vq, kp, vp, q.cpu(), pairs, new_lens, slots_of, group)
    got = out.cpu().numpy()
    for pr in pairs:
        assert_attention_close(got[pr][None], ref[pr][None])
    compare_encode(kq, kq.oracle_encode(knew.double().numpy()), *unpack(kq, kp, rows=new_slots))
    compare_encode(vq, vq.oracle_encode(vnew.double().numpy()), *unpack(vq, vp, rows=new_slots))
    return out


@pytest.mark.parametrize("kbits,km,vbits", [(2, 128, 3), (3, 128, 2), (1, 128, 3), (3, 0, 3)])
def test_decode_step_tensor_core_path(tq, kbits, km, vbits):
    """d 128, 4 query heads per KV head, token-block values: appends and query preparation in one
    launch; lengths that cross a 16-token block and a chunk boundary, and an empty sequence."""
    _step_case(tq, 128, kbits, km, vbits, 1, batch=4, hkv=2, group=4, lens=[2600, 15, 0, 511], paged=False,
               seed=301 + 10 * kbits + vbits)


def test_decode_step_tensor_core_paged_bf16(tq):
    _step_case(tq, 128, 2, 128, 3, 1, batch=3, hkv=3, group=4, lens=[700, 16, 1031], paged=True, seed=331,
               kvdtype=torch.bfloat16, qdtype=torch.float32)


@pytest.mark.parametrize("d,group,vlayout", [(64, 2, 0), (128, 8, 1), (128, 4, 0)])
def test_decode_step_general_path(tq, d, group, vlayout):
    """Shapes the tensor-core kernel does not take: the step runs the separate calls."""
    _step_case(tq, d, 2, d, 3, vlayout, batch=2, hkv=2, group=group, lens=[300, 47], paged=False,
               seed=351 + d + group)


@pytest.mark.parametrize("vlayout", [1, 0])
def test_decode_step_structured_qjl(tq, vlayout):
    """Keys with the structured QJL matrix S = P H D2: the appended key's signs come from the
    in-register Walsh-Hadamard transform, the queries are projected with the same S."""
    _step_case(tq, 128, 2, 128, 3, vlayout, batch=2, hkv=2, group=4, lens=[1500, 33], paged=vlayout == 1,
               seed=371 + vlayout, srht=True)


def test_decode_step_fp16_norms(tq):
    """tq_decode_step with norms stored in fp16: the appended rows and the attention equal the
    separate calls' and match the oracle on the library's own bytes."""
    _step_case(tq, 128, 2, 128, 3, 1, batch=3, hkv=2, group=4, lens=[700, 15, 1031], paged=True, seed=211,
               kvdtype=torch.bfloat16, norm_bits=16)
