"""Pins of the oracle's full-vocabulary top-k and Hit@k ("Cut Binary Cross
Entropy", section III-E): brute force with plain Python sorting on tiny inputs,
ties broken by the lower id, permutation of the items, chunk-size invariance,
and scikit-learn's top_k_accuracy_score for queries with one target."""
import numpy as np
import pytest

from oracle import cutbce_oracle as O


def _brute(Q, E, k):
    ids, scores = [], []
    for q in Q:
        s = [(sum(float(a) * float(b) for a, b in zip(q, e)), v) for v, e in enumerate(E)]
        s.sort(key=lambda x: (-x[0], x[1]))
        ids.append([v for _, v in s[:k]])
        scores.append([x for x, _ in s[:k]])
    return np.array(ids), np.array(scores)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force(seed):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((5, 3))
    E = rng.standard_normal((23, 3))
    ids, scores = O.topk(Q, E, 8, chunk=7)
    bi, bs = _brute(Q, E, 8)
    assert np.array_equal(ids, bi) and np.allclose(scores, bs, rtol=0, atol=1e-12)


def test_ties_prefer_the_lower_id():
    E = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 0.0], [0.5, 0.5], [1.0, 0.0]])
    Q = np.array([[2.0, 0.0], [1.0, 1.0]])
    ids, _ = O.topk(Q, E, 3, chunk=2)
    assert ids[0].tolist() == [0, 2, 4]          # three equal scores: ids ascending
    assert ids[1].tolist() == [0, 1, 2]          # all five tie at 1.0


def test_permutation_and_chunks():
    rng = np.random.default_rng(3)
    Q = rng.standard_normal((4, 8))
    E = rng.standard_normal((300, 8))
    ids, scores = O.topk(Q, E, 8)
    perm = rng.permutation(300)                  # item v of E[perm] is item perm[v] of E
    pids, pscores = O.topk(Q, E[perm], 8)
    assert np.array_equal(perm[pids], ids) and np.allclose(pscores, scores)
    for chunk in (1, 13, 300):
        assert np.array_equal(O.topk(Q, E, 8, chunk=chunk)[0], ids)


def test_hit_at_k_and_scikit_learn():
    sk = pytest.importorskip("sklearn.metrics")
    rng = np.random.default_rng(4)
    Q = rng.standard_normal((40, 6))
    E = rng.standard_normal((30, 6))
    y = rng.integers(0, 30, 40)
    ids, _ = O.topk(Q, E, 5)
    hits = O.hit_at_k(ids, y[:, None])
    ref = sk.top_k_accuracy_score(y, Q @ E.T, k=5, labels=np.arange(30))
    assert hits.mean() == pytest.approx(ref)
    # several targets, empty slots and a query with none
    tg = np.array([[ids[0, 4], -1, 7], [-1, -1, -1]] + [[-1, -1, -1]] * 38)
    h = O.hit_at_k(ids, tg)
    assert h[0] == 1 and h[1] == 0
