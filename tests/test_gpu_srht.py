"""GPU parity of the structured QJL option (tq_ctx_create_srht: S = P H D2, the first m rows of
the unnormalised Sylvester Hadamard matrix with columns times random signs D2, "TurboQuant 学习
路径" 二.2): the encode transforms the residual in registers instead of multiplying by a dense S,
and must give the oracle's sign bits (with the 1e-5 band on z) at every d and m; scores and search
then run unchanged on the dense S the context derives from D2."""
import numpy as np
import pytest
import torch

import synth
from oracle import search as osearch
from parity import (Quantizer, assert_scores_close, assert_topk_equivalent, compare_encode,
                    oracle_scores_from_packed, unpack)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_06_b200 import tq as _tq
    return _tq


def _enc(tq, q, x, slots=None, capacity=None):
    packed = tq.Packed.allocate(q.ctx, capacity or x.shape[0])
    tq.encode_kv(q.ctx, x.cuda(), packed, slots=None if slots is None else slots.cuda())
    torch.cuda.synchronize()
    return packed


@pytest.mark.parametrize("d,m", [(32, 32), (64, 32), (128, 128), (128, 64), (256, 256), (1024, 1024), (1024, 512)])
@pytest.mark.parametrize("bits", [1, 2, 3])
def test_srht_encode_matches_oracle(tq, d, m, bits):
    q = Quantizer(d, bits, m, seed=400 + d + m + bits, srht=True)
    assert tq.encode_workspace_size(q.ctx, 100000) == 0
    x = torch.randn(3001, d, generator=torch.Generator().manual_seed(d + bits)) * torch.exp(
        torch.randn(d, generator=torch.Generator().manual_seed(7)))
    packed = _enc(tq, q, x)
    stats = compare_encode(q, q.oracle_encode(x.double().numpy()), *unpack(q, packed))
    assert stats["sign_flips"] <= 1e-4 * x.shape[0] * m


def test_srht_encode_large_batch_bf16_with_slots(tq):
    """More rows than the dense path's fused limit, bf16 rows, scattered slots over stale bytes."""
    d, m = 128, 128
    q = Quantizer(d, 2, m, seed=431, srht=True)
    n = 9000
    x = (torch.randn(n, d, generator=torch.Generator().manual_seed(3)) * 3).to(torch.bfloat16)
    perm = torch.randperm(2 * n, generator=torch.Generator().manual_seed(4))[:n]
    packed = tq.Packed.allocate(q.ctx, 2 * n)
    packed.codes.fill_(0xAB)
    packed.signs.fill_(0xCD)
    tq.encode_kv(q.ctx, x.cuda(), packed, slots=perm.cuda())
    torch.cuda.synchronize()
    compare_encode(q, q.oracle_encode(x.double().numpy()), *unpack(q, packed, rows=perm.numpy()))


def test_srht_scores_and_search(tq):
    """The Tiny workload's shape with the structured matrix: scores through the estimator, and
    top-10 search on the tcgen05 (40 queries) and mma.sync (8 queries) scans."""
    keys, queries = synth.tiny(seed=0)
    q = Quantizer(128, 2, 128, seed=441, srht=True)
    packed = _enc(tq, q, keys)
    codes, sbits, norm, rnorm = unpack(q, packed)
    got = tq.scores(q.ctx, queries.cuda(), packed).cpu().numpy()
    ref = oracle_scores_from_packed(q, queries.double().numpy(), codes, sbits, norm, rnorm)
    assert_scores_close(got, ref)
    for nq in (8, 40):
        Q = synth.unit_rows(nq, 128, seed=442 + nq)
        s, i = tq.search_topk(q.ctx, Q.cuda(), packed, 10)
        torch.cuda.synchronize()
        ref_full = oracle_scores_from_packed(q, Q.double().numpy(), codes, sbits, norm, rnorm)
        ref_s, _ = osearch.topk(ref_full, 10)
        assert_topk_equivalent(s.cpu().numpy(), i.cpu().numpy(), lambda r, idx: ref_full[r, idx], ref_s)
