"""The allocation-free attention entry point, tq_attend_decode_noalloc, through the C ABI.

It serves callers that cannot allocate device memory when they run attention (an engine that
owns every byte of device memory through its own pool, or a decode loop that must never hit the
allocator).  Its scratch is the library's fixed 8 MiB device array instead of a caller workspace.
These checks compare it with tq_attend_decode (which takes a workspace) on two calls in a row —
the second call sees the first call's leftovers in the shared array — and check that an
oversized request is refused with a clear error.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oattn
from parity import Quantizer, assert_attention_close

pytestmark = pytest.mark.gpu


def _cache(tq, d, hkv, lens, paged, seed, vlayout=0):
    kq = Quantizer(d, 2, d, seed=seed)
    vq = Quantizer(d, 3, 0, seed=seed + 1, layout=vlayout)
    batch, maxlen = len(lens), int(max(lens))
    lens_t = torch.tensor(lens, dtype=torch.int32)
    table = None
    if paged:
        table, nblocks = synth.shuffled_block_table(lens_t, seed=seed + 2)
        cap = nblocks * hkv * synth.BLOCK_TOKENS
    else:
        cap = batch * hkv * maxlen
    K = synth.channel_scaled(batch, hkv, maxlen, d, seed=seed + 3)
    V = synth.channel_scaled(batch, hkv, maxlen, d, seed=seed + 4)
    slots, kx, vx = [], [], []
    for b in range(batch):
        for h in range(hkv):
            slots.append(oattn.token_slots(b, h, lens[b], hkv, ctx_stride=maxlen,
                                           block_table=None if table is None else table.numpy()))
            kx.append(K[b, h, :lens[b]])
            vx.append(V[b, h, :lens[b]])
    sl = torch.as_tensor(np.concatenate(slots), dtype=torch.int64).cuda()
    kp, vp = tq.Packed.allocate(kq.ctx, cap), tq.Packed.allocate(vq.ctx, cap)
    tq.encode_kv(kq.ctx, torch.cat(kx).cuda(), kp, slots=sl)
    tq.encode_kv(vq.ctx, torch.cat(vx).cuda(), vp, slots=sl)
    return kq, vq, kp, vp, lens_t.cuda(), maxlen, None if table is None else table.cuda()


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("vlayout", [0, 1])
def test_noalloc_matches_workspace_entry_point_twice(paged, vlayout):
    """vlayout 0: values in rows (the general CUDA-core attention); 1: values in 16-token blocks
    (the tensor-core attention, whose per-call counters live in the scratch array too)."""
    from kv_cache_vector_06_b200 import tq
    d, hkv, group = 128, 4, 4
    lens = [2500, 700, 1] if paged else [3008, 1234]
    kq, vq, kp, vp, lens_t, maxlen, table = _cache(tq, d, hkv, lens, paged, seed=71 + int(paged),
                                                   vlayout=vlayout)
    desc = tq.make_attn_desc(kq.ctx, vq.ctx, (len(lens), hkv * group, d), kp, vp, lens_t, maxlen,
                             ctx_stride=maxlen, block_table=table, block_size=synth.BLOCK_TOKENS,
                             n_kv_heads=hkv)
    assert tq.attend_workspace_size(kq.ctx, vq.ctx, desc) <= tq.NOALLOC_SCRATCH_BYTES
    for call in range(2):
        q = synth.decode_queries(len(lens), hkv * group, d, seed=100 + call).cuda()
        ref = tq.attend_decode(kq.ctx, vq.ctx, q, kp, vp, lens_t, maxlen, n_kv_heads=hkv, desc=desc)
        out = torch.full_like(ref, float("nan"))
        tq.attend_decode_noalloc(kq.ctx, vq.ctx, q, out, desc)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert_attention_close(out.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_rejects_requests_larger_than_its_scratch():
    from kv_cache_vector_06_b200 import tq
    d, hkv, group, batch, maxlen = 128, 8, 4, 300, 16
    kq = Quantizer(d, 2, d, seed=5)
    vq = Quantizer(d, 3, 0, seed=6)
    kp, vp = tq.Packed.allocate(kq.ctx, 16), tq.Packed.allocate(vq.ctx, 16)
    lens = torch.ones(batch, dtype=torch.int32, device="cuda")
    desc = tq.make_attn_desc(kq.ctx, vq.ctx, (batch, hkv * group, d), kp, vp, lens, maxlen, ctx_stride=maxlen,
                             n_kv_heads=hkv)
    assert tq.attend_workspace_size(kq.ctx, vq.ctx, desc) > tq.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(batch, hkv * group, d, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(batch, hkv * group, d, dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TqError) as e:
        tq.attend_decode_noalloc(kq.ctx, vq.ctx, q, out, desc)
    assert e.value.status == 1 and "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
