"""Pins for oracle.search: top-k selection and recall ([JJ] 第三部分 "向量搜索").

Independent references: numpy's stable argsort on small inputs, hand-made ties, the full score
matrix against the chunked scan, and recall of the exact scores.
"""
import numpy as np
import pytest

from oracle import codebook, encode, estimate, search


def test_topk_matches_stable_sort():
    rng = np.random.default_rng(0)
    sc = rng.standard_normal((6, 300))
    v, i = search.topk(sc, 10)
    for r in range(6):
        order = np.argsort(-sc[r], kind="stable")[:10]
        assert i[r].tolist() == order.tolist()
        np.testing.assert_array_equal(v[r], sc[r, order])


def test_topk_ties_go_to_lower_index():
    sc = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, 0.5]])
    v, i = search.topk(sc, 4)
    assert i[0].tolist() == [1, 2, 4, 3]
    assert v[0].tolist() == [3.0, 3.0, 3.0, 2.0]


def test_chunked_search_equals_full_scores():
    d, bits, m, n = 64, 2, 64, 5000
    rng = np.random.default_rng(1)
    X = rng.standard_normal((n, d))
    Q = rng.standard_normal((4, d))
    D = rng.choice([-1.0, 1.0], size=d)
    S = rng.standard_normal((m, d))
    c, t = codebook.codebook(d, bits)
    e = encode.encode(X, D, S, c, t)
    full = estimate.score_encoded(Q, e, D, S, c)
    v_ref, i_ref = search.topk(full, 10)
    v, i = search.search_topk(Q, e.norm, e.codes, e.rnorm, e.bits, D, S, c, 10, chunk=777)
    np.testing.assert_array_equal(i, i_ref)
    np.testing.assert_allclose(v, v_ref, rtol=1e-13)


def test_exact_topk_and_recall():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((3000, 32))
    Q = rng.standard_normal((5, 32))
    v, i = search.exact_topk(Q, X, 10, chunk=1000)
    for r in range(5):
        assert i[r].tolist() == np.argsort(-(X @ Q[r]), kind="stable")[:10].tolist()
    assert search.recall_at_k(i, i) == 1.0
    assert search.recall_at_k(i[:, ::-1], i) == 1.0


@pytest.mark.parametrize("bits,expect", [(1, 0.15), (3, 0.6)])
def test_turboquant_recall_on_unit_vectors(bits, expect):
    # Database and queries drawn N(0, I) and L2-normalised ([JJ] 第三部分 reports recall 1@k);
    # 2 and 4 bits per coordinate = (1 or 3 MSE bits) + 1 QJL bit with m = d.
    d, n = 256, 20000
    rng = np.random.default_rng(3)
    X = rng.standard_normal((n, d))
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    Q = rng.standard_normal((20, d))
    Q /= np.linalg.norm(Q, axis=1, keepdims=True)
    D = rng.choice([-1.0, 1.0], size=d)
    S = rng.standard_normal((d, d))
    c, t = codebook.codebook(d, bits)
    e = encode.encode(X, D, S, c, t)
    _, i = search.search_topk(Q, e.norm, e.codes, e.rnorm, e.bits, D, S, c, 10)
    _, ie = search.exact_topk(Q, X, 10)
    assert search.recall_at_k(i, ie) > expect


def test_recall_hand_counted():
    # two queries, k = 4: 3 of 4 exact neighbours found, then 1 of 4 (order inside a list and the
    # extra wrong entries do not matter): recall = (3/4 + 1/4) / 2 = 0.5
    exact = [[7, 1, 5, 2], [10, 11, 12, 13]]
    found = [[1, 2, 9, 7], [13, 3, 4, 8]]
    assert search.recall_at_k(found, exact) == 0.5
    assert search.recall_at_k([[1, 2, 9, 7]], [[7, 1, 5, 2]]) == 0.75
    # a found list longer than k (k is the exact list's length): hits / k, not hits / len(found)
    assert search.recall_at_k([[7, 1, 5, 2, 99, 98]], [[7, 1, 5, 2]]) == 1.0
    assert search.recall_at_k([[0, 0, 0, 0]], [[7, 1, 5, 2]]) == 0.0
