"""GPU parity at the full workload sizes, in the launch configuration bench.py times.

The oracle cannot form the whole [T, V] problem of these workloads in seconds,
so each output is compared with oracle values it can compute:

  * the loss over the whole vocabulary against the float64 oracle's full sum,
    written once by tests/golden/make_fullv_loss.py (oracle only);
  * dH on at least 512 valid positions: all of the first and of the last
    128-position tile, plus a seeded random set, each row formed by the oracle
    from its own logit row;
  * dE on at least 1,024 items: the 256 most frequent positive ids (the Zipf
    head), the first and last row of every 32nd 128-item tile, the whole last
    (ragged) tile, plus seeded random items, each row formed by the oracle from
    its own logit column;
  * three item slices of 8,192 items against the oracle's loss on that slice.

The relative Frobenius error over the sampled rows must stay within the
tolerance of the full comparison (2e-3); the loss within 1e-5 relative.
"""
import json
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import binding as B
from vocabulary_label_bce_b200 import workloads as W
from gpu_util import GRAD_RTOL, LOSS_RTOL, rel_fro, to_device

pytestmark = pytest.mark.gpu

ORACLE_SLICE = 8192    # items per slice compared with the oracle's slice loss
N_DH_ROWS = 512
N_DE_ROWS = 1024
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "fullv_loss.json")


def _golden(name):
    with open(GOLDEN) as f:
        entries = {e["workload"]: e for e in json.load(f)["entries"]}
    return entries[name]


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


def _in_threads(fn, groups):
    """Run fn on each group in a thread pool (numpy releases the interpreter lock
    inside its array kernels) with one BLAS thread per pool thread; results in
    group order."""
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1, "blas")
    except ImportError:  # pragma: no cover
        limit = None
    try:
        with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
            return list(ex.map(fn, groups))
    finally:
        if limit is not None:
            limit.unregister()


def _split(xs, n):
    return [xs[i::n] for i in range(n) if xs[i::n]]


def sampled_positions(p, rng):
    valid = np.nonzero(p.mask)[0]
    nv = len(valid)
    first = valid[:128].tolist()
    last = valid[(nv - 1) // 128 * 128:].tolist()
    chosen = set(first) | set(last)
    rest = np.setdiff1d(valid, np.array(sorted(chosen)))
    extra = rng.choice(rest, max(0, N_DH_ROWS - len(chosen)), replace=False).tolist()
    return sorted(chosen | set(extra))


def sampled_items(p, rng):
    valid_tg = p.targets[p.mask != 0]
    ids = valid_tg[valid_tg >= 0].astype(np.int64)
    counts = np.bincount(ids, minlength=p.V)
    hottest = np.lexsort((np.arange(p.V), -counts))[:256].tolist()   # most frequent, lower id first
    n_tiles = (p.V + 127) // 128
    edges = []
    for k in range(0, n_tiles, 32):
        edges += [128 * k, min(p.V - 1, 128 * k + 127)]
    last_tile = list(range((p.V - 1) // 128 * 128, p.V))
    chosen = set(hottest) | set(edges) | set(last_tile)
    if len(chosen) < N_DE_ROWS:
        pool = np.setdiff1d(np.arange(p.V), np.array(sorted(chosen)))
        chosen |= set(rng.choice(pool, N_DE_ROWS - len(chosen), replace=False).tolist())
    return sorted(chosen)


@pytest.mark.parametrize("name", ["sasrec_876k", "wide_d256", "extreme_10m"])
def test_full_size_sampled(name):
    gold = _golden(name)
    p = W.draw_config(name, seed=gold["seed"])
    assert (p.T, p.V, p.D, p.K) == (gold["T"], gold["V"], gold["D"], gold["K"])
    H, E, tg, m = to_device(p)
    prob, ws, loss_mean, dH, dE = _call(H, E, tg, m, "mean")

    # integer side results are exact
    rc = torch.empty(p.T, dtype=torch.int32)
    nv, npairs = B.cutbce_read_counts(prob, ws, rc)
    tgs = O.positive_sets(p.targets, p.mask, p.V)
    assert nv == tgs.n_valid == gold["n_valid"] and npairs == tgs.n_pairs == gold["n_pairs"]
    assert np.array_equal(rc.numpy(), tgs.row_counts.astype(np.int32))

    # the loss over the whole vocabulary against the oracle's full sum
    err_loss = abs(loss_mean - gold["mean_loss"]) / abs(gold["mean_loss"])
    assert err_loss <= LOSS_RTOL, (loss_mean, gold["mean_loss"], err_loss)

    rng = np.random.default_rng(1)
    items = sampled_items(p, rng)
    pos = sampled_positions(p, rng)
    assert len(items) >= N_DE_ROWS and len(pos) >= N_DH_ROWS
    got_dE = dE[torch.tensor(items, device=dE.device)].double().cpu().numpy()
    got_dH = dH[torch.tensor(pos, device=dH.device)].double().cpu().numpy()
    masked = np.nonzero(p.mask == 0)[0]
    if len(masked):
        assert torch.all(dH[torch.tensor(masked, device=dH.device)] == 0)
    del dH, dE
    torch.cuda.empty_cache()

    ref_dE = np.concatenate(_in_threads(lambda g: O.dE_rows(p.H, p.E, p.targets, p.mask, g),
                                        _split(items, 64)))
    order_dE = np.concatenate(_split(items, 64))
    ref_dE = ref_dE[np.argsort(order_dE)]
    ref_dH = np.concatenate(_in_threads(lambda g: O.dH_rows(p.H, p.E, p.targets, p.mask, g),
                                        _split(pos, 16)))
    order_dH = np.concatenate(_split(pos, 16))
    ref_dH = ref_dH[np.argsort(order_dH)]
    err_dE = rel_fro(got_dE, ref_dE)
    err_dH = rel_fro(got_dH, ref_dH)
    print(name, {"loss_rel": err_loss, "dE_rel_sampled": err_dE, "dE_rows": len(items),
                 "dH_rel_sampled": err_dH, "dH_rows": len(pos)})
    assert err_dE <= GRAD_RTOL and err_dH <= GRAD_RTOL

    # item slices against the oracle's slice loss (reduction SUM)
    for v0 in (0, (p.V // 2) // 128 * 128, (p.V - ORACLE_SLICE) // 128 * 128):
        v1 = min(p.V, v0 + ORACLE_SLICE)
        _, _, got, _, _ = _call(H, E[v0:v1], _slice_targets(tg, v0, v1), m, "sum", want_grad=False)
        ref = O.loss_sum_slice(p.H, p.E, p.targets, p.mask, v0, v1)
        assert abs(got - ref) <= LOSS_RTOL * abs(ref), (v0, got, ref)
