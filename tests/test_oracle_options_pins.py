"""Pins of the oracle's per-position weights and vocabulary shards.

Weights (the `weights` argument of the paper's API, "Cut Binary Cross Entropy"
section III-C Listing 1): all-ones weights and {0, 1} weights must reproduce the
unweighted and the masked results exactly; central finite differences and
torch's binary_cross_entropy_with_logits(weight=...) with autograd fix the
weighted loss and both gradients.  Shards: the loss sums, the dH rows and the
Cut Metrics of a vocabulary cut into shards must add up to the unsharded ones,
and the dE rows of the shards must be the unsharded rows (additivity of
Eqs. (2)-(4) over the items)."""
import numpy as np
import pytest
import torch

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import workloads as W


def _problem(seed=0, T=9, V=23, D=4, K=5):
    rng = np.random.default_rng(seed)
    H = rng.standard_normal((T, D))
    E = rng.standard_normal((V, D)) * 0.8
    targets = rng.integers(-1, V, size=(T, K)).astype(np.int32)
    mask = np.ones(T, dtype=np.uint8)
    mask[2] = 0
    w = rng.uniform(0.2, 2.0, size=T)
    w[5] = 0.0
    w[7] = -0.5                                   # negative weights are allowed
    return H, E, targets, mask, w


def test_unit_weights_and_zero_one_weights():
    p = W.draw(T=50, V=400, D=16, K=6, dtype="bf16", seed=1, ids="zipf", mask="random", mask_frac=0.2)
    for red in (O.MEAN_VALID_POSITIONS, O.SUM, O.MEAN_ELEMENTS):
        a = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=red)
        b = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=red, weights=np.ones(p.T))
        assert a.loss == b.loss and np.array_equal(a.dH, b.dH) and np.array_equal(a.dE, b.dE)
        c = O.forward_backward(p.H, p.E, p.targets, None, reduction=red, weights=p.mask.astype(np.float64))
        assert a.loss == c.loss and np.array_equal(a.dH, c.dH) and np.array_equal(a.dE, c.dE)
        assert a.n_valid == c.n_valid


def test_weighted_finite_differences():
    H, E, targets, mask, w = _problem()
    r = O.forward_backward(H, E, targets, mask, reduction=O.SUM, weights=w)
    h = 1e-6
    for (A, G) in ((H, r.dH), (E, r.dE)):
        num = np.zeros_like(A)
        for idx in np.ndindex(A.shape):
            Ap, Am = A.copy(), A.copy()
            Ap[idx] += h
            Am[idx] -= h
            args = (Ap, E) if A is H else (H, Ap)
            argm = (Am, E) if A is H else (H, Am)
            lp = O.forward_backward(*args, targets, mask, reduction=O.SUM, weights=w, want_grad=False).loss
            lm = O.forward_backward(*argm, targets, mask, reduction=O.SUM, weights=w, want_grad=False).loss
            num[idx] = (lp - lm) / (2 * h)
        assert np.max(np.abs(num - G)) <= 1e-6 * max(1.0, np.max(np.abs(G)))


@pytest.mark.parametrize("red", [O.MEAN_VALID_POSITIONS, O.SUM])
def test_weighted_against_torch(red):
    H, E, targets, mask, w = _problem(seed=3)
    r = O.forward_backward(H, E, targets, mask, reduction=red, weights=w, grad_loss=0.7)
    Ht = torch.tensor(H, requires_grad=True)
    Et = torch.tensor(E, requires_grad=True)
    valid = (mask != 0) & (w != 0)
    Y = np.zeros((H.shape[0], E.shape[0]))
    for t in range(H.shape[0]):
        if valid[t]:
            Y[t, targets[t][targets[t] >= 0]] = 1.0
    wt = torch.tensor(np.where(valid, w, 0.0))[:, None].expand(H.shape[0], E.shape[0])
    loss = torch.nn.functional.binary_cross_entropy_with_logits(Ht @ Et.T, torch.tensor(Y), weight=wt,
                                                                reduction="sum")
    if red == O.MEAN_VALID_POSITIONS:
        loss = loss / int(valid.sum())
    (0.7 * loss).backward()
    assert r.loss == pytest.approx(float(loss), rel=1e-12)
    assert np.allclose(r.dH, Ht.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(r.dE, Et.grad.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("red", [O.MEAN_VALID_POSITIONS, O.SUM, O.MEAN_ELEMENTS])
def test_vocabulary_shards_add_up(red):
    p = W.draw(T=40, V=333, D=8, K=6, dtype="f32", seed=4, ids="zipf", mask="random", mask_frac=0.1)
    w = np.random.default_rng(5).uniform(0.5, 1.5, p.T)
    full = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=red, weights=w)
    fullm = O.cut_metrics(p.H, p.E, p.targets, p.mask, weights=w)
    cuts = [0, 100, 101, 250, p.V]
    loss, dH, dE, met = 0.0, np.zeros_like(full.dH), [], np.zeros_like(fullm)
    for v0, v1 in zip(cuts[:-1], cuts[1:]):
        r = O.forward_backward(p.H, p.E[v0:v1], p.targets, p.mask, reduction=red, weights=w, vocab_offset=v0,
                               V_total=p.V)
        loss += r.loss
        dH += r.dH
        dE.append(r.dE)
        met += O.cut_metrics(p.H, p.E[v0:v1], p.targets, p.mask, weights=w, vocab_offset=v0, V_total=p.V)
        assert r.n_valid == full.n_valid
    assert loss == pytest.approx(full.loss, rel=1e-12)
    assert np.allclose(dH, full.dH, rtol=1e-12, atol=1e-14)
    assert np.allclose(np.concatenate(dE), full.dE, rtol=1e-12, atol=1e-14)
    assert np.array_equal(met, fullm)


def test_shard_id_rules():
    H, E, _, mask, _ = _problem(seed=6, V=10)
    targets = np.random.default_rng(7).integers(-1, 30, size=(H.shape[0], 6)).astype(np.int32)
    r = O.forward_backward(H, E, targets, mask, vocab_offset=10, V_total=30)
    expect = [len(np.unique(row[(row >= 10) & (row < 20)])) if mask[t] else 0 for t, row in enumerate(targets)]
    assert r.row_counts.tolist() == expect                      # ids of other shards are dropped, not errors
    targets[1, 0] = 30                                          # outside the whole vocabulary: an error
    with pytest.raises(O.TargetRangeError):
        O.forward_backward(H, E, targets, mask, vocab_offset=10, V_total=30)
