"""Inner-product top-k search over the compressed database, and exact brute force (fp64).

Source.
  [JJ] 第三部分 "向量搜索": TurboQuant is a general vector quantizer; nearest-neighbour search by
       inner product over compressed vectors, evaluated by recall 1@k against exact search.
  [JJ] 第五部分 "对向量搜索的影响": the same scoring serves retrieval.

Definitions (R = reading):
  score(q, x_i) is the estimator of oracle.estimate.
  top-k orders by (score descending, index ascending) (R: ties go to the lower index).
  recall@k = |found ∩ exact| / k averaged over queries, exact = fp64 brute force on the
  uncompressed vectors.

Pinned by tests/test_oracle_search.py: equals a full sort on small inputs, ties resolve to the
lower index, chunked selection equals one-shot selection, recall of exact scores is 1.
"""
from __future__ import annotations

import numpy as np

from .estimate import prepare_query, scores


def topk(sc, k: int):
    """Row-wise top-k of a score matrix [nq, n] -> (scores [nq, k], idx [nq, k])."""
    sc = np.asarray(sc, dtype=np.float64)
    nq, n = sc.shape
    idx = np.empty((nq, k), dtype=np.int64)
    val = np.empty((nq, k))
    ar = np.arange(n)
    for i in range(nq):
        order = np.lexsort((ar, -sc[i]))[:k]
        idx[i] = order
        val[i] = sc[i, order]
    return val, idx


def search_topk(q, norm, codes, rnorm, bits, signs, S, centroids, k: int, chunk: int = 65536):
    """Top-k of the estimated scores of queries q [nq, d] against a database given as unpacked
    arrays; the database is processed in row chunks and the candidates re-selected."""
    qr, p = prepare_query(q, signs, S)
    n = len(norm)
    best_v = None
    best_i = None
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        sc = scores(qr, p, norm[s:e], codes[s:e], rnorm[s:e], bits[s:e], centroids)
        v, i = topk(sc, min(k, e - s))
        i = i + s
        if best_v is None:
            best_v, best_i = v, i
        else:
            cv = np.concatenate([best_v, v], axis=1)
            ci = np.concatenate([best_i, i], axis=1)
            keep_v = np.empty((cv.shape[0], k))
            keep_i = np.empty((cv.shape[0], k), dtype=np.int64)
            for r in range(cv.shape[0]):
                order = np.lexsort((ci[r], -cv[r]))[:k]
                keep_v[r] = cv[r, order]
                keep_i[r] = ci[r, order]
            best_v, best_i = keep_v, keep_i
    return best_v, best_i


def exact_topk(q, X, k: int, chunk: int = 65536):
    """Exact fp64 inner-product top-k (brute force)."""
    q = np.asarray(q, dtype=np.float64)
    n = X.shape[0]
    best_v = None
    best_i = None
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        sc = q @ np.asarray(X[s:e], dtype=np.float64).T
        v, i = topk(sc, min(k, e - s))
        i = i + s
        if best_v is None:
            best_v, best_i = v, i
        else:
            cv = np.concatenate([best_v, v], axis=1)
            ci = np.concatenate([best_i, i], axis=1)
            order = [np.lexsort((ci[r], -cv[r]))[:k] for r in range(cv.shape[0])]
            best_v = np.stack([cv[r, o] for r, o in enumerate(order)])
            best_i = np.stack([ci[r, o] for r, o in enumerate(order)])
    return best_v, best_i


def recall_at_k(found_idx, exact_idx) -> float:
    found_idx = np.asarray(found_idx)
    exact_idx = np.asarray(exact_idx)
    k = exact_idx.shape[1]
    hits = [len(set(found_idx[i].tolist()) & set(exact_idx[i].tolist())) for i in range(len(exact_idx))]
    return float(np.mean(hits)) / k
