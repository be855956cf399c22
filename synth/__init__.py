"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the benchmark.

This module only draws numbers.  It holds none of the quantizer's arithmetic: no rotation,
no codebook, no packing, no estimator.  The random quantities that the method itself draws
(the rotation's sign vector D and the Gaussian JL matrix S) are produced here as plain inputs,
so that the oracle and the CUDA library receive identical values and neither has to
re-implement a random number generator.

Every generator uses a torch CPU generator seeded explicitly, so the values are identical
across runs and machines.  bf16 inputs are drawn in fp32 and rounded once to bf16; the oracle
receives the rounded values widened to fp64.
"""
from __future__ import annotations

import torch

BLOCK_TOKENS = 16  # tokens per paged KV block


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


# ----------------------------------------------------------------------------- method draws
def rotation_signs(d: int, seed: int) -> torch.Tensor:
    """D: d independent fair +-1 signs (int8)."""
    g = _gen(seed)
    return (torch.randint(0, 2, (d,), generator=g, dtype=torch.int8) * 2 - 1).to(torch.int8)


def qjl_matrix(m: int, d: int, seed: int) -> torch.Tensor:
    """S: m x d matrix of iid N(0,1) entries, fp32, row-major."""
    if m == 0:
        return torch.zeros(0, d, dtype=torch.float32)
    g = _gen(seed)
    return torch.randn(m, d, generator=g, dtype=torch.float32)


# ----------------------------------------------------------------------------- workloads
def tiny(seed: int = 0, n: int = 4096, d: int = 128, nq: int = 8, n_outlier: int = 4,
         outlier_scale: float = 20.0):
    """One head: n fp32 keys iid N(0,1) with channels 0..n_outlier-1 scaled (outliers),
    nq fp32 queries iid N(0,1)."""
    g = _gen(seed)
    keys = torch.randn(n, d, generator=g, dtype=torch.float32)
    keys[:, :n_outlier] *= outlier_scale
    queries = torch.randn(nq, d, generator=g, dtype=torch.float32)
    return keys, queries


def channel_scaled(batch: int, n_kv: int, ctx: int, d: int, seed: int,
                   dtype=torch.bfloat16) -> torch.Tensor:
    """[batch, n_kv, ctx, d] = N(0,1) * s[kv head, channel], s ~ lognormal(0, 1), then one
    rounding to `dtype`.  Call once for K and once for V with different seeds."""
    g = _gen(seed)
    scale = torch.exp(torch.randn(n_kv, d, generator=g, dtype=torch.float32))
    out = torch.empty(batch, n_kv, ctx, d, dtype=dtype)
    # draw per (batch, head) so memory stays bounded for long contexts
    for b in range(batch):
        for h in range(n_kv):
            x = torch.randn(ctx, d, generator=g, dtype=torch.float32) * scale[h]
            out[b, h] = x.to(dtype)
    return out


def decode_queries(batch: int, n_q: int, d: int, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """[batch, n_q, d] iid N(0,1), rounded to `dtype`."""
    g = _gen(seed)
    return torch.randn(batch, n_q, d, generator=g, dtype=torch.float32).to(dtype)


def unit_rows(n: int, d: int, seed: int, chunk: int = 65536) -> torch.Tensor:
    """[n, d] fp32 rows drawn N(0, I) and then L2-normalised (search database / queries)."""
    g = _gen(seed)
    out = torch.empty(n, d, dtype=torch.float32)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = torch.randn(e - s, d, generator=g, dtype=torch.float64)
        x /= x.norm(dim=1, keepdim=True)
        out[s:e] = x.to(torch.float32)
    return out


def ragged_lengths(batch: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """Per-sequence context lengths, uniform integers in [lo, hi] (int32)."""
    g = _gen(seed)
    return torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int64).to(torch.int32)


def shuffled_block_table(ctx_lens: torch.Tensor, seed: int, block_tokens: int = BLOCK_TOKENS):
    """Assign every sequence ceil(len/block_tokens) physical blocks drawn from one seeded
    permutation of all blocks.  Returns (block_table int32 [batch, max_blocks] padded with 0,
    total number of physical blocks)."""
    nblk = [(int(n) + block_tokens - 1) // block_tokens for n in ctx_lens.tolist()]
    total = sum(nblk)
    g = _gen(seed)
    perm = torch.randperm(total, generator=g).to(torch.int32)
    width = max(nblk) if nblk else 0
    table = torch.zeros(len(nblk), max(width, 1), dtype=torch.int32)
    o = 0
    for b, k in enumerate(nblk):
        table[b, :k] = perm[o:o + k]
        o += k
    return table, total


def bf16_round(x: torch.Tensor) -> torch.Tensor:
    """Round fp32 values to bf16 and back (for inputs the pages store in bf16)."""
    return x.to(torch.bfloat16).to(torch.float32)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [
    "BLOCK_TOKENS", "rotation_signs", "qjl_matrix", "tiny", "channel_scaled", "decode_queries",
    "unit_rows", "ragged_lengths", "shuffled_block_table", "bf16_round", "ceil_div"
]
