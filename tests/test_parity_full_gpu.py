"""GPU parity at the full workload sizes, in the launch configuration bench.py times.

The oracle cannot form the whole [T, V] problem at these sizes in seconds, so:
  * dE is compared on sampled item rows (the Zipf head item 0, items of the
    ragged last tile, random items), each computed by the oracle one by one;
  * dH is compared on sampled positions (plus a masked one, which must be 0);
  * the loss is pinned by additivity over the vocabulary: the GPU's full summed
    loss equals the sum of its losses on item slices aligned to item tiles,
    and sampled slices equal the oracle's loss on the same slice.
"""
import numpy as np
import pytest
import torch

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import binding as B
from vocabulary_label_bce_b200 import workloads as W
from gpu_util import GRAD_RTOL, LOSS_RTOL, rel_fro, to_device

pytestmark = pytest.mark.gpu

SLICE = 65536          # items per slice for the additivity check (a multiple of the 128-item tile)
ORACLE_SLICE = 8192    # items per slice compared with the oracle


def _call(H, E, tg, m, reduction, want_grad=True):
    prob = B.make_problem(H, E, tg, m, reduction)
    ws = torch.empty(B.cutbce_workspace_size(prob), dtype=torch.uint8, device=H.device)
    loss = torch.empty((), dtype=torch.float64, device=H.device)
    dH = torch.empty(H.shape, dtype=torch.float32, device=H.device) if want_grad else None
    dE = torch.empty(E.shape, dtype=torch.float32, device=H.device) if want_grad else None
    B.cutbce_forward_backward(prob, None, loss, dH, dE, ws)
    assert B.cutbce_read_status(ws) == 0
    return prob, ws, float(loss.item()), dH, dE


def _slice_targets(tg, v0, v1):
    inside = (tg >= v0) & (tg < v1)
    return torch.where(inside, tg - v0, torch.full_like(tg, -1)).contiguous()


@pytest.mark.parametrize("name", ["sasrec_876k", "wide_d256", "extreme_10m"])
def test_full_size_sampled(name):
    p = W.draw_config(name, seed=0)
    H, E, tg, m = to_device(p)
    prob, ws, loss_mean, dH, dE = _call(H, E, tg, m, "mean")

    # integer side results are exact
    rc = torch.empty(p.T, dtype=torch.int32)
    nv, npairs = B.cutbce_read_counts(prob, ws, rc)
    tgs = O.positive_sets(p.targets, p.mask, p.V)
    assert nv == tgs.n_valid and npairs == tgs.n_pairs
    assert np.array_equal(rc.numpy(), tgs.row_counts.astype(np.int32))

    rng = np.random.default_rng(1)
    last_tile = (p.V - 1) // 128 * 128
    items = sorted(set([0, 1, 2, 127, 128, p.V - 1, last_tile] + list(rng.integers(0, p.V, 17))))
    ref_dE = O.dE_rows(p.H, p.E, p.targets, p.mask, items)
    got_dE = dE[torch.tensor(items, device=dE.device)].double().cpu().numpy()
    err_dE = rel_fro(got_dE, ref_dE)
    valid = np.nonzero(p.mask)[0]
    masked = np.nonzero(p.mask == 0)[0]
    pos = sorted(set([int(valid[0]), int(valid[-1])] + list(rng.choice(valid, 6, replace=False))))
    ref_dH = O.dH_rows(p.H, p.E, p.targets, p.mask, pos)
    got_dH = dH[torch.tensor(pos, device=dH.device)].double().cpu().numpy()
    err_dH = rel_fro(got_dH, ref_dH)
    if len(masked):
        assert torch.all(dH[torch.tensor(masked[:64], device=dH.device)] == 0)
    print(name, {"dE_rel_sampled": err_dE, "dH_rel_sampled": err_dH})
    assert err_dE <= GRAD_RTOL and err_dH <= GRAD_RTOL
    del dH, dE

    # loss: additivity over item slices, and sampled slices against the oracle
    _, _, full_sum, _, _ = _call(H, E, tg, m, "sum", want_grad=False)
    parts = 0.0
    for v0 in range(0, p.V, SLICE):
        v1 = min(p.V, v0 + SLICE)
        _, _, part, _, _ = _call(H, E[v0:v1], _slice_targets(tg, v0, v1), m, "sum", want_grad=False)
        parts += part
    assert abs(parts - full_sum) <= 1e-9 * abs(full_sum), (parts, full_sum)
    assert abs(loss_mean * nv - full_sum) <= 1e-9 * abs(full_sum)
    for v0 in (0, (p.V // 2) // 128 * 128, (p.V - ORACLE_SLICE) // 128 * 128):
        v1 = min(p.V, v0 + ORACLE_SLICE)
        _, _, got, _, _ = _call(H, E[v0:v1], _slice_targets(tg, v0, v1), m, "sum", want_grad=False)
        ref = O.loss_sum_slice(p.H, p.E, p.targets, p.mask, v0, v1)
        assert abs(got - ref) <= LOSS_RTOL * abs(ref), (v0, got, ref)
