"""Shared helpers for the GPU parity tests: build matching oracle/library quantizers from the same
seeded draws, and compare library outputs with the oracle under the tolerances of the method's
conformance contract:

  codes / sign bits : bit-exact, except entries whose pre-quantization value lies within 1e-5 of
                      a threshold (unit rotated domain for codes, z = <s, r> for signs); the count
                      of such mismatches must stay under 1e-4 of the entries
  scores            : |gpu - ref| <= max(1e-4, 1e-3 |ref|)
  attention         : ||gpu - ref||_inf <= 2e-3 ||ref||_inf per (sequence, head)
  top-k             : identical up to ties within 1e-6
"""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import attention as oattn
from oracle import codebook as ocb
from oracle import encode as oenc
from oracle import estimate as oest

BAND = 1e-5
MAX_FLIP_FRACTION = 1e-4


class Quantizer:
    """One tensor role: the seeded draws (D, S), the oracle codebook and the library context."""

    def __init__(self, d, bits, m, seed, device=0, layout=0, srht=False, norm_bits=32):
        """srht: structured QJL, S = P H D2 with D2 drawn like D (the oracle builds S, the library
        receives only D2).  norm_bits: 32 or 16, the storage of the norms."""
        from kv_cache_vector_06_b200 import tq
        self.d, self.bits, self.m, self.layout, self.norm_bits = d, bits, m, layout, norm_bits
        self.D = synth.rotation_signs(d, seed)
        self.c, self.t = ocb.codebook(d, bits)
        if srht:
            self.D2 = synth.rotation_signs(d, seed + 2000)
            self.S = torch.from_numpy(oenc.srht_matrix(self.D2.double().numpy(), m))
            self.ctx = tq.Context(d, bits, m, self.D, device=device, layout=layout, qjl_signs=self.D2,
                                  norm_bits=norm_bits)
        else:
            self.S = synth.qjl_matrix(m, d, seed + 1000)
            self.ctx = tq.Context(d, bits, m, self.D, self.S if m > 0 else None, device=device, layout=layout,
                                  norm_bits=norm_bits)

    @property
    def D64(self):
        return self.D.double().numpy()

    @property
    def S64(self):
        return self.S.double().numpy()

    def oracle_encode(self, x64):
        return oenc.store_norms(oenc.encode(x64, self.D64, self.S64, self.c, self.t), self.norm_bits)


def unpack(q: Quantizer, packed, rows=None):
    """Library packed arrays (torch, device) -> unpacked numpy (codes, bits, norm, rnorm)."""
    sel = slice(None) if rows is None else torch.as_tensor(rows, device=packed.codes.device)
    if q.layout == 1:   # token-block layout: decode the 16-slot blocks that hold the rows
        cb = packed.codes.shape[1]
        if rows is None:
            codes = oenc.unpack_codes_block16(packed.codes.cpu().numpy(), q.d, q.bits)
        else:
            r = np.asarray(torch.as_tensor(rows).cpu()).astype(np.int64)
            blocks = np.unique(r // 16)
            blk = packed.codes.view(-1, 16, cb)[torch.as_tensor(blocks, device=packed.codes.device)]
            dec = oenc.unpack_codes_block16(blk.reshape(-1, cb).cpu().numpy(), q.d, q.bits)
            codes = dec[np.searchsorted(blocks, r // 16) * 16 + r % 16]
    else:
        codes = oenc.unpack_codes(packed.codes[sel].cpu().numpy(), q.d, q.bits)
    norm = packed.norm[sel].double().cpu().numpy()
    if q.m > 0:
        bits = oenc.unpack_signs(packed.signs[sel].cpu().numpy(), q.m)
        rnorm = packed.rnorm[sel].double().cpu().numpy()
    else:
        bits = np.zeros((codes.shape[0], 0), dtype=np.uint8)
        rnorm = np.zeros(codes.shape[0])
    return codes, bits, norm, rnorm


def compare_encode(q: Quantizer, enc: "oenc.Encoded", codes, bits, norm, rnorm):
    """Check library encodings against the oracle's; returns a dict of counts."""
    n = codes.shape[0]
    # fp16 norms: the library rounds its fp32 norm, the oracle its fp64 one: one half ulp apart at most
    nrt = 2e-6 if q.norm_bits == 32 else 2.0 ** -10
    np.testing.assert_allclose(norm, enc.norm, rtol=nrt, atol=1e-30)
    near_thr = np.min(np.abs(enc.y[:, :, None] - q.t[None, None, :]), axis=2) < BAND
    code_bad = codes != enc.codes
    assert not np.any(code_bad & ~near_thr), "code mismatch outside the threshold band"
    flips = int(code_bad.sum())
    assert flips <= max(1, MAX_FLIP_FRACTION * codes.size), f"{flips} code flips"
    rows_ok = ~code_bad.any(axis=1)
    sign_flips = 0
    if q.m > 0:
        near0 = np.abs(enc.z) < BAND
        bad = (bits != enc.bits) & rows_ok[:, None]
        assert not np.any(bad & ~near0), "sign mismatch outside the |z| < 1e-5 band"
        sign_flips = int(bad.sum())
        assert sign_flips <= max(1, MAX_FLIP_FRACTION * bits.size), f"{sign_flips} sign flips"
        np.testing.assert_allclose(rnorm[rows_ok], enc.rnorm[rows_ok], rtol=max(2e-5, nrt), atol=1e-6)
    return {"n": n, "code_flips": flips, "sign_flips": sign_flips}


def assert_scores_close(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    tol = np.maximum(1e-4, 1e-3 * np.abs(ref))
    err = np.abs(got - ref)
    assert np.all(err <= tol), f"max excess {np.max(err - tol)} (max err {np.max(err)})"


def assert_attention_close(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    for idx in np.ndindex(ref.shape[:-1]):
        r = ref[idx]
        if np.any(np.isnan(r)):
            continue
        lim = 2e-3 * np.max(np.abs(r))
        e = np.max(np.abs(got[idx] - r))
        assert e <= lim or (lim == 0 and e == 0), f"{idx}: err {e} > {lim}"


def assert_topk_equivalent(gpu_scores, gpu_idx, ref_scores_full_fn, ref_top_scores, tie=1e-6):
    """gpu_idx [nq, k]; ref_scores_full_fn(i, idx) -> oracle scores of query i at rows idx;
    ref_top_scores [nq, k] oracle's sorted top-k scores."""
    nq, k = gpu_idx.shape
    for i in range(nq):
        s_of_gpu = ref_scores_full_fn(i, gpu_idx[i])
        assert len(set(gpu_idx[i].tolist())) == k, "duplicate indices"
        tol = tie + tie * np.abs(ref_top_scores[i])
        assert np.all(np.abs(s_of_gpu - ref_top_scores[i]) <= tol), (i, s_of_gpu, ref_top_scores[i])
        assert_scores_close(gpu_scores[i], s_of_gpu)


def oracle_cache(q: Quantizer, codes, bits, norm, rnorm):
    if q.m > 0:
        return oattn.Cache(norm=norm, codes=codes, rnorm=rnorm, bits=bits)
    return oattn.Cache(norm=norm, codes=codes)


def oracle_scores_from_packed(q: Quantizer, queries64, codes, bits, norm, rnorm):
    qr, p = oest.prepare_query(queries64, q.D64, q.S64)
    return oest.scores(qr, p, norm, codes, rnorm, bits, q.c)


def oracle_heads(kq, vq, kp, vp, q, pairs, lens, slots_fn, group):
    """Oracle attention output for sampled (sequence, query head) pairs, decoding only the slots of
    each pair's KV head from the library's packed arrays.  q: torch [B, Hq, d]."""
    out = {}
    for b, hq in pairs:
        h = hq // group
        L = int(lens[b])
        sl = np.asarray(slots_fn(b, h, L), dtype=np.int64)
        kc = oracle_cache(kq, *unpack(kq, kp, rows=sl))
        vc = oracle_cache(vq, *unpack(vq, vp, rows=sl))
        r = oattn.attend_decode(q[b, hq][None, None].double().cpu().numpy(), kc, vc, [L], 1, kq.D64, kq.S64, kq.c,
                                vq.D64, vq.c, ctx_stride=L)
        out[(b, hq)] = r[0, 0]
    return out
