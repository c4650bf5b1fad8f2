"""Pins of the oracle's Cut Metrics ("Cut Binary Cross Entropy", section III-D):
per-position TP, FP, FN, TN over the whole vocabulary, item v predicted positive
iff sigmoid(x_tv) > 1/2 (x_tv > 0).

Tied to facts other than the oracle itself: brute-force enumeration with plain
Python loops on tiny inputs, the identities TP + FP + FN + TN = V and
TP + FN = |P_t|, the closed form at H = 0, invariance under permuting the items,
chunk-size invariance, and scikit-learn's accuracy, precision, recall and F_beta
on the dense 0/1 predictions.  A swapped FP/FN, a >= instead of >, a dropped
mask or a transposed operand fails at least one of them."""
import numpy as np
import pytest

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import workloads as W


def _brute(H, E, targets, mask):
    T, V = H.shape[0], E.shape[0]
    out = np.zeros((T, 4), dtype=np.int64)
    for t in range(T):
        if mask is not None and mask[t] == 0:
            continue
        pos = {int(v) for v in targets[t] if v >= 0}
        for v in range(V):
            z = sum(float(H[t, d]) * float(E[v, d]) for d in range(H.shape[1]))
            p = z > 0.0
            y = v in pos
            out[t, 0 if (p and y) else 1 if p else 2 if y else 3] += 1
    return out


def _tiny(seed, T=7, V=16, D=3, K=4):
    rng = np.random.default_rng(seed)
    H = rng.standard_normal((T, D))
    E = rng.standard_normal((V, D))
    targets = rng.integers(-1, V, size=(T, K)).astype(np.int32)
    targets[0, :2] = targets[0, 2]                   # repeated ids count once
    mask = np.ones(T, dtype=np.uint8)
    mask[T // 2] = 0
    targets[T // 2, 0] = 10 * V                       # ignored: the row is masked
    return H, E, targets, mask


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_brute_force(seed):
    H, E, targets, mask = _tiny(seed)
    assert np.array_equal(O.cut_metrics(H, E, targets, mask, chunk=5), _brute(H, E, targets, mask))


def test_exact_zero_logit_is_a_predicted_negative():
    # integer-valued inputs make several logits exactly 0
    H = np.array([[1.0, -1.0], [2.0, 0.0], [0.0, 0.0]])
    E = np.array([[1.0, 1.0], [0.0, 3.0], [-1.0, 2.0], [1.0, 0.0]])
    targets = np.array([[0, 1], [1, -1], [2, 3]], dtype=np.int32)
    got = O.cut_metrics(H, E, targets, None)
    assert np.array_equal(got, _brute(H, E, targets, None))
    # row 0: z = (0, -3, -3, 1): positives {0, 1} -> TP 0, FN 2; predicted positive {3} -> FP 1
    assert got[0].tolist() == [0, 1, 2, 1]


def test_identities_and_masked_rows():
    p = W.draw(T=40, V=300, D=16, K=6, dtype="bf16", seed=4, ids="zipf", mask="random", mask_frac=0.2)
    c = O.cut_metrics(p.H, p.E, p.targets, p.mask)
    tg = O.positive_sets(p.targets, p.mask, p.V)
    valid = p.mask != 0
    assert np.all(c[~valid] == 0)
    assert np.all(c[valid].sum(axis=1) == p.V)
    assert np.array_equal(c[:, 0] + c[:, 2], tg.row_counts)


def test_zero_activations_closed_form():
    p = W.draw(T=30, V=200, D=8, K=5, dtype="bf16", seed=5, mask="random", mask_frac=0.1)
    H0 = np.zeros_like(p.H)
    c = O.cut_metrics(H0, p.E, p.targets, p.mask)
    tg = O.positive_sets(p.targets, p.mask, p.V)
    valid = p.mask != 0
    assert np.all(c[:, 0] == 0) and np.all(c[:, 1] == 0)
    assert np.array_equal(c[valid, 2], tg.row_counts[valid])
    assert np.array_equal(c[valid, 3], p.V - tg.row_counts[valid])


def test_item_permutation_and_chunk_invariance():
    p = W.draw(T=25, V=257, D=8, K=4, dtype="f32", seed=6, ids="uniform", mask="none")
    base = O.cut_metrics(p.H, p.E, p.targets, None)
    perm = np.random.default_rng(7).permutation(p.V)          # new id of old item v is inv[v]
    inv = np.argsort(perm)
    tg2 = np.where(p.targets >= 0, inv[np.maximum(p.targets, 0)], -1).astype(np.int32)
    assert np.array_equal(O.cut_metrics(p.H, p.E[perm], tg2, None), base)
    for chunk in (1, 64, p.V):
        assert np.array_equal(O.cut_metrics(p.H, p.E, p.targets, None, chunk=chunk), base)


def test_metrics_match_scikit_learn():
    sk = pytest.importorskip("sklearn.metrics")
    p = W.draw(T=20, V=150, D=8, K=10, dtype="f32", seed=8, e_std=0.6, ids="uniform", mask="random", mask_frac=0.1)
    c = O.cut_metrics(p.H, p.E, p.targets, p.mask)
    valid = p.mask != 0
    Z = p.H[valid].astype(np.float64) @ p.E.astype(np.float64).T
    y_pred = (Z > 0).ravel()
    Y = np.zeros_like(Z, dtype=bool)
    for r, t in enumerate(np.nonzero(valid)[0]):
        Y[r, p.targets[t][p.targets[t] >= 0]] = True
    y_true = Y.ravel()
    m = O.metrics_from_counts(c, beta=0.5)
    assert m["accuracy"] == pytest.approx(sk.accuracy_score(y_true, y_pred), abs=1e-12)
    assert m["precision"] == pytest.approx(sk.precision_score(y_true, y_pred, zero_division=0), abs=1e-12)
    assert m["recall"] == pytest.approx(sk.recall_score(y_true, y_pred, zero_division=0), abs=1e-12)
    assert m["fbeta"] == pytest.approx(sk.fbeta_score(y_true, y_pred, beta=0.5, zero_division=0), abs=1e-12)
