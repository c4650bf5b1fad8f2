"""Cut Metrics on the GPU ("Cut Binary Cross Entropy", section III-D) against the
float64 oracle: per-position TP, FP, FN, TN over the whole vocabulary.

The kernel decides x > 0 on its fp32 accumulation of the bf16 products; the
oracle decides on the exact float64 logit.  The two can differ only where the
exact logit lies within the fp32 accumulation error of 0, so each element with
|x| <= 2^-16 * sum_d |h_d e_d| (far above that error for D <= 256) counts as
undecided: a row's TP (FP) may move by at most its undecided positives
(negatives) and FN (TN) with it.  Rows with no undecided element must match
exactly, and TP + FP + FN + TN = V, TP + FN = |P_t| hold exactly everywhere."""
import numpy as np
import pytest
import torch

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import binding as B
from vocabulary_label_bce_b200 import workloads as W
from gpu_util import GRAD_RTOL, LOSS_RTOL, rel_fro, to_device

pytestmark = pytest.mark.gpu

TIE_REL = 2.0 ** -16


def undecided(p, chunk=4096):
    """Per position: undecided positives and undecided negatives (elements near x = 0)."""
    tg = O.positive_sets(p.targets, p.mask, p.V)
    out = np.zeros((p.T, 2), dtype=np.int64)
    rows = np.nonzero(tg.valid)[0]
    H = p.H[rows].astype(np.float64)
    for c0 in range(0, p.V, chunk):
        c1 = min(p.V, c0 + chunk)
        E = p.E[c0:c1].astype(np.float64)
        near = np.abs(H @ E.T) <= TIE_REL * (np.abs(H) @ np.abs(E).T)
        if not near.any():
            continue
        for r, t in enumerate(rows):
            if near[r].any():
                cols = np.nonzero(near[r])[0] + c0
                pos = np.isin(cols, tg.sets[t])
                out[t, 0] += int(pos.sum())
                out[t, 1] += int((~pos).sum())
    return out


def check_metrics(p, got):
    ref = O.cut_metrics(p.H, p.E, p.targets, p.mask)
    tg = O.positive_sets(p.targets, p.mask, p.V)
    valid = p.mask != 0
    assert np.all(got[~valid] == 0)
    assert np.all(got[valid].sum(axis=1) == p.V)
    assert np.array_equal(got[:, 0] + got[:, 2], tg.row_counts)
    und = undecided(p)
    exact = und.sum(axis=1) == 0
    assert np.array_equal(got[exact], ref[exact]), np.nonzero((got != ref).any(axis=1) & exact)[0][:10]
    assert np.all(np.abs(got[:, 0] - ref[:, 0]) <= und[:, 0])
    assert np.all(np.abs(got[:, 1] - ref[:, 1]) <= und[:, 1])
    return int((~exact & valid).sum())


def run_ex(p, want_loss, want_dH, want_dE, tensors=None):
    H, E, tg, m = tensors if tensors is not None else to_device(p)
    prob = B.make_problem(H, E, tg, m, "mean")
    bits = B.OUT_METRICS | (B.OUT_LOSS if want_loss else 0) | (B.OUT_DH if want_dH else 0) | \
        (B.OUT_DE if want_dE else 0)
    ws = torch.empty(B.cutbce_workspace_size_for(prob, bits), dtype=torch.uint8, device="cuda")
    met = torch.full((p.T, 4), -7, dtype=torch.int32, device="cuda")
    loss = torch.full((), float("nan"), dtype=torch.float64, device="cuda") if want_loss else None
    dH = torch.full((p.T, p.D), float("nan"), dtype=torch.float32, device="cuda") if want_dH else None
    dE = torch.full((p.V, p.D), float("nan"), dtype=torch.float32, device="cuda") if want_dE else None
    B.cutbce_forward_backward_ex(prob, B.make_options(metrics=met), None, loss, dH, dE, ws)
    assert B.cutbce_read_status(ws) == 0
    return {"metrics": met.cpu().numpy().astype(np.int64),
            "loss": float(loss.item()) if loss is not None else None,
            "dH": dH.cpu().numpy() if dH is not None else None,
            "dE": dE.cpu().numpy() if dE is not None else None}


SHAPES = [
    dict(T=300, V=1000, D=64, K=5),
    dict(T=257, V=2047, D=128, K=8),
    dict(T=200, V=777, D=256, K=16),
    dict(T=130, V=515, D=192, K=6),
    dict(T=100, V=300, D=32, K=4),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"T{s['T']}_V{s['V']}_D{s['D']}")
@pytest.mark.parametrize("mode", ["metrics_only", "with_dH", "all"])
def test_metrics_match_oracle(shape, mode):
    p = W.draw(**shape, dtype="bf16", seed=21, ids="zipf", zipf_s=1.1, mask="random", mask_frac=0.1)
    got = run_ex(p, mode == "all", mode != "metrics_only", mode == "all")
    n_und = check_metrics(p, got["metrics"])
    print(shape, mode, "rows with undecided elements:", n_und)
    if mode != "metrics_only":
        ref = O.forward_backward(p.H, p.E, p.targets, p.mask)
        assert rel_fro(got["dH"], ref.dH) <= GRAD_RTOL
        if mode == "all":
            assert abs(got["loss"] - ref.loss) <= LOSS_RTOL * abs(ref.loss)
            assert rel_fro(got["dE"], ref.dE) <= GRAD_RTOL


def test_metrics_saturated_logits_and_zero_rows():
    # the paper's stress distribution (|x| up to ~40) plus rows of H that are exactly 0,
    # whose logits are all exactly 0: every item is a predicted negative there
    p = W.draw(T=256, V=2000, D=128, K=8, dtype="bf16", seed=22, e_std=1.0, ids="uniform", mask="random",
               mask_frac=0.1)
    p.H[::17] = 0
    p.H_bits[::17] = 0
    got = run_ex(p, True, True, True)
    check_metrics(p, got["metrics"])
    tg = O.positive_sets(p.targets, p.mask, p.V)
    for t in range(0, p.T, 17):
        if p.mask[t]:
            assert got["metrics"][t].tolist() == [0, 0, int(tg.row_counts[t]), p.V - int(tg.row_counts[t])]


def test_metrics_small_catalog():
    p = W.draw_config("small_catalog")
    got = run_ex(p, False, True, False)
    check_metrics(p, got["metrics"])


def test_metrics_fp32_path():
    p = W.draw_config("tiny_f32")
    got = run_ex(p, True, True, True)
    check_metrics(p, got["metrics"])


def test_metrics_do_not_change_the_other_outputs():
    p = W.draw(T=333, V=1500, D=64, K=4, dtype="bf16", seed=23, ids="zipf", mask="random", mask_frac=0.2)
    t = to_device(p)
    a = run_ex(p, True, True, True, tensors=t)
    H, E, tg, m = t
    prob = B.make_problem(H, E, tg, m, "mean")
    ws = torch.empty(B.cutbce_workspace_size(prob), dtype=torch.uint8, device="cuda")
    loss = torch.empty((), dtype=torch.float64, device="cuda")
    dH = torch.empty((p.T, p.D), dtype=torch.float32, device="cuda")
    dE = torch.empty((p.V, p.D), dtype=torch.float32, device="cuda")
    B.cutbce_forward_backward(prob, None, loss, dH, dE, ws)
    assert float(loss.item()) == a["loss"]
    assert np.array_equal(dH.cpu().numpy(), a["dH"]) and np.array_equal(dE.cpu().numpy(), a["dE"])
