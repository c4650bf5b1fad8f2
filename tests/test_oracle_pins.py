"""Pins of the float64 oracle to things other than itself.

Each test ties the oracle to a fact fixed by the mathematics ("Cut Binary
Cross Entropy", section III-A Eqs. (1)-(3), section III-B Eq. (4)) or by an
independent implementation: the literal Eq. (1), closed forms at H = 0 and
E = 0, central finite differences, torch's own binary_cross_entropy_with_logits
with autograd, and invariances that any correct implementation must satisfy.
A dropped term, a wrong sign, a transposed operand or a wrong normalisation in
the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import workloads as W


def _tiny_fd_problem():
    # T=4, V=7, D=3 with a duplicate id, a -1 slot and a masked row.
    rng = np.random.default_rng(123)
    H = rng.standard_normal((4, 3))
    E = rng.standard_normal((7, 3)) * 0.7
    targets = np.array([[2, 5, 2, -1],
                        [0, -1, -1, -1],
                        [6, 1, 3, 3],
                        [4, 4, -1, 0]], dtype=np.int32)
    mask = np.array([1, 1, 0, 1], dtype=np.uint8)
    return H, E, targets, mask


def _torch_reference(H, E, targets, mask, reduction, grad_loss=1.0):
    """Dense BCE with torch's own BCE-with-logits in float64, gradients by autograd."""
    V = E.shape[0]
    Ht = torch.tensor(np.asarray(H, dtype=np.float64), requires_grad=True)
    Et = torch.tensor(np.asarray(E, dtype=np.float64), requires_grad=True)
    valid = np.asarray(mask) != 0 if mask is not None else np.ones(H.shape[0], bool)
    Y = np.zeros((H.shape[0], V))
    for t in range(H.shape[0]):
        if valid[t]:
            ids = targets[t][targets[t] >= 0]
            Y[t, ids] = 1.0
    w = torch.tensor(valid.astype(np.float64))[:, None]
    Z = Ht @ Et.T
    per = torch.nn.functional.binary_cross_entropy_with_logits(
        Z, torch.tensor(Y), reduction="none") * w
    n_valid = int(valid.sum())
    total = per.sum()
    if n_valid == 0:
        loss = total * 0.0
    elif reduction == O.SUM:
        loss = total
    elif reduction == O.MEAN_VALID_POSITIONS:
        loss = total / n_valid
    else:
        loss = total / (n_valid * V)
    (loss * grad_loss).backward()
    return float(loss), Ht.grad.numpy(), Et.grad.numpy()


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(np.linalg.norm(b), 1e-300)
    return np.linalg.norm(a - b) / den


# ---------------------------------------------------------------- element identities
def test_eq1_equals_eq2_moderate_range():
    x = np.linspace(-8, 8, 4001)
    for y in (0.0, 1.0):
        a = O.bce_eq1(x, np.full_like(x, y))
        b = O.bce_eq2(x, np.full_like(x, y))
        # Eq. (1) taken literally loses ~eps/(1-s(x)) to cancellation; 1e-11 covers |x| <= 8
        assert np.max(np.abs(a - b) / np.maximum(np.abs(b), 1e-300)) < 1e-11


def test_eq2_identities():
    x = np.linspace(-60, 60, 2401)
    sp = O.bce_eq2(x, np.zeros_like(x))             # softplus(x)
    # BCE(x, 1) = softplus(x) - x
    np.testing.assert_allclose(O.bce_eq2(x, np.ones_like(x)), sp - x, rtol=0, atol=1e-13)
    # softplus(x) - softplus(-x) = x
    np.testing.assert_allclose(sp - O.bce_eq2(-x, np.zeros_like(x)), x, rtol=0, atol=1e-12)
    # exact value at 0 and known values log(1+e^x)
    assert O.bce_eq2(np.array([0.0]), np.array([0.0]))[0] == pytest.approx(math.log(2.0), abs=1e-16)
    assert O.bce_eq2(np.array([math.log(3.0)]), np.array([0.0]))[0] == pytest.approx(math.log(4.0), rel=1e-15)
    assert O.bce_eq2(np.array([-math.log(3.0)]), np.array([0.0]))[0] == pytest.approx(math.log(4.0 / 3.0), rel=1e-15)
    assert np.all(np.isfinite(O.bce_eq2(np.array([-1e4, 1e4]), np.array([1.0, 0.0]))))


def test_sigmoid_branches_and_symmetry():
    x = np.linspace(-700, 700, 14001)
    s = O.sigmoid(x)
    np.testing.assert_allclose(s + O.sigmoid(-x), 1.0, atol=1e-15)
    assert O.sigmoid(np.array([0.0]))[0] == 0.5
    assert O.sigmoid(np.array([math.log(3.0)]))[0] == pytest.approx(0.75, rel=1e-15)
    # derivative of softplus is the sigmoid (central difference)
    xs = np.linspace(-6, 6, 121)
    h = 1e-6
    fd = (O.bce_eq2(xs + h, 0 * xs) - O.bce_eq2(xs - h, 0 * xs)) / (2 * h)
    np.testing.assert_allclose(fd, O.sigmoid(xs), atol=1e-9)


# ---------------------------------------------------------------- target rules
def test_positive_sets_rules():
    targets = np.array([[3, 3, -1, 0], [5, -1, -1, -1], [9, 9, 9, 9], [-1, -1, -1, -1]], np.int32)
    mask = np.array([1, 1, 0, 1], np.uint8)
    tg = O.positive_sets(targets, mask, V=6)           # row 2 is masked: its ids (9 >= V) are ignored
    assert tg.n_valid == 3
    assert [list(s) for s in tg.sets] == [[0, 3], [5], [], []]
    assert list(tg.row_counts) == [2, 1, 0, 0]
    assert tg.n_pairs == 3
    with pytest.raises(O.TargetRangeError):
        O.positive_sets(np.array([[6]], np.int32), None, V=6)
    with pytest.raises(O.TargetRangeError):
        O.positive_sets(np.array([[-2]], np.int32), None, V=6)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("zero", ["H", "E"])
def test_closed_form_zero_operand(zero):
    p = W.draw(T=40, V=300, D=16, K=5, dtype="bf16", seed=7, ids="uniform",
               mask="random", mask_frac=0.2)
    H, E = p.H.astype(np.float64), p.E.astype(np.float64)
    if zero == "H":
        H = np.zeros_like(H)
    else:
        E = np.zeros_like(E)
    r = O.forward_backward(H, E, p.targets, p.mask, reduction=O.SUM)
    tg = O.positive_sets(p.targets, p.mask, p.V)
    # every logit is 0: each element costs ln 2 and the target correction y*x vanishes
    assert r.sum_loss == pytest.approx(tg.n_valid * p.V * math.log(2.0), rel=1e-14)
    if zero == "H":
        assert np.all(r.dE == 0.0)
        for t in range(p.T):
            want = np.zeros(p.D) if not tg.valid[t] else 0.5 * E.sum(0) - E[tg.sets[t]].sum(0)
            np.testing.assert_allclose(r.dH[t], want, rtol=1e-12, atol=1e-12)
    else:
        assert np.all(r.dH == 0.0)
        hs = (H * tg.valid[:, None]).sum(0)
        for v in range(p.V):
            want = 0.5 * hs - sum((H[t] for t in range(p.T) if tg.valid[t] and v in tg.sets[t]),
                                  np.zeros(p.D))
            np.testing.assert_allclose(r.dE[v], want, rtol=1e-12, atol=1e-12)


def test_single_element_by_hand():
    # T=1, V=2, D=1: x = (ln 3, -ln 3), item 0 positive.
    H = np.array([[1.0]])
    E = np.array([[math.log(3.0)], [-math.log(3.0)]])
    r = O.forward_backward(H, E, np.array([[0, -1]], np.int32), None, reduction=O.SUM)
    # l(ln3, 1) = ln(4/3); l(-ln3, 0) = ln(4/3)
    assert r.loss == pytest.approx(2 * math.log(4.0 / 3.0), rel=1e-14)
    # G = (3/4 - 1, 1/4) ; dH = G.E = -1/4 ln3 - 1/4 ln3 ; dE = G^T H
    assert r.dH[0, 0] == pytest.approx(-0.5 * math.log(3.0), rel=1e-14)
    np.testing.assert_allclose(r.dE[:, 0], [-0.25, 0.25], rtol=1e-14)


# ---------------------------------------------------------------- finite differences
@pytest.mark.parametrize("reduction", [O.SUM, O.MEAN_VALID_POSITIONS, O.MEAN_ELEMENTS])
def test_finite_differences(reduction):
    H, E, targets, mask = _tiny_fd_problem()
    r = O.forward_backward(H, E, targets, mask, reduction=reduction, grad_loss=1.0)
    h = 1e-6

    def loss(Hx, Ex):
        return O.forward_backward(Hx, Ex, targets, mask, reduction=reduction, want_grad=False).loss

    gH = np.zeros_like(H)
    for idx in np.ndindex(H.shape):
        Hp, Hm = H.copy(), H.copy()
        Hp[idx] += h
        Hm[idx] -= h
        gH[idx] = (loss(Hp, E) - loss(Hm, E)) / (2 * h)
    gE = np.zeros_like(E)
    for idx in np.ndindex(E.shape):
        Ep, Em = E.copy(), E.copy()
        Ep[idx] += h
        Em[idx] -= h
        gE[idx] = (loss(H, Ep) - loss(H, Em)) / (2 * h)
    assert _rel(r.dH, gH) < 1e-7
    assert _rel(r.dE, gE) < 1e-7
    assert np.all(r.dH[2] == 0.0)                      # masked row


# ---------------------------------------------------------------- independent library
@pytest.mark.parametrize("reduction", [O.SUM, O.MEAN_VALID_POSITIONS, O.MEAN_ELEMENTS])
def test_torch_bce_with_logits_fd_case(reduction):
    H, E, targets, mask = _tiny_fd_problem()
    r = O.forward_backward(H, E, targets, mask, reduction=reduction, grad_loss=0.37)
    l_ref, gH, gE = _torch_reference(H, E, targets, mask, reduction, grad_loss=0.37)
    assert r.loss == pytest.approx(l_ref, rel=1e-12)
    assert _rel(r.dH, gH) < 1e-12
    assert _rel(r.dE, gE) < 1e-12


def test_torch_bce_with_logits_tiny_config():
    p = W.draw_config("tiny_f32")
    for reduction in (O.SUM, O.MEAN_VALID_POSITIONS):
        r = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=reduction, chunk=300)
        l_ref, gH, gE = _torch_reference(p.H, p.E, p.targets, p.mask, reduction)
        assert r.loss == pytest.approx(l_ref, rel=1e-12)
        assert _rel(r.dH, gH) < 1e-12
        assert _rel(r.dE, gE) < 1e-12


def test_stress_paper_distribution():
    # A, E ~ N(0, I), D=128, L=8 uniform ids (mini-benchmark inputs): |x| reaches ~40.
    p = W.draw(T=48, V=900, D=128, K=8, dtype="bf16", seed=3, e_std=1.0, ids="uniform", mask="none")
    r = O.forward_backward(p.H, p.E, p.targets, None, reduction=O.SUM, chunk=256)
    assert np.isfinite(r.loss) and np.all(np.isfinite(r.dH)) and np.all(np.isfinite(r.dE))
    Z = p.H.astype(np.float64) @ p.E.astype(np.float64).T
    assert np.abs(Z).max() > 30
    l_ref, gH, gE = _torch_reference(p.H, p.E, p.targets, None, O.SUM)
    assert r.loss == pytest.approx(l_ref, rel=1e-12)
    assert _rel(r.dH, gH) < 1e-11
    assert _rel(r.dE, gE) < 1e-11


# ---------------------------------------------------------------- invariances
def test_chunk_size_invariance():
    p = W.draw(T=30, V=257, D=8, K=4, dtype="bf16", seed=11, ids="zipf", zipf_s=1.1,
               mask="random", mask_frac=0.1)
    base = O.forward_backward(p.H, p.E, p.targets, p.mask, chunk=p.V)
    for c in (1, 7, 8192):
        r = O.forward_backward(p.H, p.E, p.targets, p.mask, chunk=c)
        assert r.loss == pytest.approx(base.loss, rel=1e-12)
        assert _rel(r.dH, base.dH) < 1e-12
        assert _rel(r.dE, base.dE) < 1e-12


def test_normalisation_modes_and_empty():
    p = W.draw(T=20, V=50, D=8, K=3, dtype="bf16", seed=5, mask="random", mask_frac=0.25)
    s = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=O.SUM)
    m = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=O.MEAN_VALID_POSITIONS, grad_loss=2.0)
    e = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=O.MEAN_ELEMENTS)
    nv = p.n_valid
    assert m.loss == pytest.approx(s.loss / nv, rel=1e-14)
    assert e.loss == pytest.approx(s.loss / (nv * p.V), rel=1e-14)
    np.testing.assert_allclose(m.dH, 2.0 * s.dH / nv, rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(e.dE, s.dE / (nv * p.V), rtol=1e-13, atol=1e-300)
    z = O.forward_backward(p.H, p.E, p.targets, np.zeros(p.T, np.uint8))
    assert z.loss == 0.0 and np.all(z.dH == 0) and np.all(z.dE == 0)


def test_masking_equals_deletion_and_duplicates_collapse():
    p = W.draw(T=25, V=64, D=8, K=4, dtype="bf16", seed=9, mask="random", mask_frac=0.2)
    r = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=O.SUM)
    keep = p.mask != 0
    d = O.forward_backward(p.H[keep], p.E, p.targets[keep], None, reduction=O.SUM)
    assert r.loss == pytest.approx(d.loss, rel=1e-14)
    np.testing.assert_allclose(r.dH[keep], d.dH, rtol=1e-13)
    np.testing.assert_allclose(r.dE, d.dE, rtol=1e-13, atol=1e-15)
    dup = p.targets.copy()
    dup[:, -1] = dup[:, 0]                      # repeat an id already present in the row
    r2 = O.forward_backward(p.H, p.E, dup, p.mask, reduction=O.SUM)
    r3 = O.forward_backward(p.H, p.E, _dedup_rows(dup), p.mask, reduction=O.SUM)
    assert r2.loss == r3.loss
    assert np.array_equal(r2.dH, r3.dH) and np.array_equal(r2.dE, r3.dE)


def _dedup_rows(t):
    out = np.full_like(t, -1)
    for i, row in enumerate(t):
        u = []
        for x in row:
            if x >= 0 and x not in u:
                u.append(int(x))
        out[i, :len(u)] = u
    return out


def test_item_permutation_invariance():
    p = W.draw(T=16, V=40, D=8, K=3, dtype="bf16", seed=21)
    r = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=O.SUM)
    perm = np.random.default_rng(0).permutation(p.V)       # new id of old item v is inv[v]
    inv = np.argsort(perm)
    E2 = p.E[perm]
    t2 = np.where(p.targets >= 0, inv[np.maximum(p.targets, 0)], -1).astype(np.int32)
    r2 = O.forward_backward(p.H, E2, t2, p.mask, reduction=O.SUM)
    assert r2.loss == pytest.approx(r.loss, rel=1e-13)
    np.testing.assert_allclose(r2.dH, r.dH, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r2.dE, r.dE[perm], rtol=1e-12, atol=1e-14)


def test_row_samplers_agree_with_dense():
    p = W.draw(T=33, V=515, D=16, K=5, dtype="bf16", seed=4, ids="zipf", mask="random", mask_frac=0.1)
    r = O.forward_backward(p.H, p.E, p.targets, p.mask, grad_loss=0.5)
    items = [0, 1, 2, 100, 514]
    np.testing.assert_allclose(O.dE_rows(p.H, p.E, p.targets, p.mask, items, grad_loss=0.5),
                               r.dE[items], rtol=1e-12, atol=1e-15)
    pos = list(range(p.T))
    np.testing.assert_allclose(O.dH_rows(p.H, p.E, p.targets, p.mask, pos, grad_loss=0.5, chunk=100),
                               r.dH, rtol=1e-12, atol=1e-15)
    parts = sum(O.loss_sum_slice(p.H, p.E, p.targets, p.mask, a, min(p.V, a + 128), chunk=50)
                for a in range(0, p.V, 128))
    assert parts == pytest.approx(r.sum_loss, rel=1e-13)


def test_regression_fixture():
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_regression.json")
    ref = json.load(open(path))
    p = W.draw(**ref["problem"])
    for case in ref["cases"]:
        r = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=case["reduction"],
                               grad_loss=case["grad_loss"])
        assert r.loss == pytest.approx(case["loss"], rel=1e-13)
        assert r.n_valid == case["n_valid"] and r.n_pairs == case["n_pairs"]
        np.testing.assert_allclose(r.dH.sum(1), case["dH_row_sums"], rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(r.dE[:3], case["dE_first_rows"], rtol=1e-12, atol=1e-15)
