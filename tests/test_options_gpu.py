"""The options of cutbce_forward_backward_ex on the GPU against the float64
oracle: per-position weights ("Cut Binary Cross Entropy", section III-C Listing
1), bf16 gradient outputs, accumulation into dH / dE, and vocabulary shards.

bf16 outputs are the round-to-nearest-even of the call's fp32 result, and
accumulation adds in fp32 and rounds once, so both are checked bit for bit
against the fp32 outputs of the same call; weights and shards are checked
against the oracle at the usual tolerances, and the integer side results
(which positions and pairs contribute) bit for bit."""
import numpy as np
import pytest
import torch

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import binding as B
from vocabulary_label_bce_b200 import workloads as W
from gpu_util import GRAD_RTOL, LOSS_RTOL, RED, rel_fro, to_device

pytestmark = pytest.mark.gpu


def call(p, tensors, reduction="mean", want=("loss", "dH", "dE"), weights=None, metrics=False,
         grad_dtype=B.GRAD_F32, accumulate=0, init=None, vocab_offset=0, V_total=0, E=None, tg=None):
    H, E0, tg0, m = tensors
    E = E0 if E is None else E
    tg = tg0 if tg is None else tg
    prob = B.make_problem(H, E, tg, m, reduction)
    dt = torch.bfloat16 if grad_dtype == B.GRAD_BF16 else torch.float32
    met = torch.full((p.T, 4), -7, dtype=torch.int32, device="cuda") if metrics else None
    w = torch.from_numpy(np.asarray(weights, dtype=np.float32)).cuda() if weights is not None else None
    opts = B.make_options(metrics=met, weights=w, grad_dtype=grad_dtype, accumulate=accumulate,
                          vocab_offset=vocab_offset, V_total=V_total)
    bits = (B.OUT_LOSS if "loss" in want else 0) | (B.OUT_DH if "dH" in want else 0) | \
        (B.OUT_DE if "dE" in want else 0) | (B.OUT_METRICS if metrics else 0)
    ws = torch.empty(B.cutbce_workspace_size_ex(prob, opts, bits), dtype=torch.uint8, device="cuda")
    loss = torch.full((), float("nan"), dtype=torch.float64, device="cuda") if "loss" in want else None
    dH = dE = None
    if "dH" in want:
        dH = init[0].clone() if init is not None else torch.full((p.T, p.D), float("nan"), dtype=dt, device="cuda")
    if "dE" in want:
        dE = init[1].clone() if init is not None else torch.full((E.shape[0], p.D), float("nan"), dtype=dt,
                                                                 device="cuda")
    B.cutbce_forward_backward_ex(prob, opts, None, loss, dH, dE, ws)
    st = B.cutbce_read_status(ws)
    assert st == 0, B.cutbce_status_string(st)
    rc = torch.empty(p.T, dtype=torch.int32)
    nv, npairs = B.cutbce_read_counts(prob, ws, rc)
    return {"loss": float(loss.item()) if loss is not None else None, "dH": dH, "dE": dE,
            "metrics": met.cpu().numpy().astype(np.int64) if met is not None else None,
            "n_valid": nv, "n_pairs": npairs, "row_counts": rc.numpy()}


def weights_for(p, seed):
    w = np.random.default_rng(seed).uniform(0.25, 2.0, p.T).astype(np.float32)
    w[::11] = 0.0                      # padding by weight
    w[5::13] = -0.75                   # negative weights are allowed
    return w


SHAPES = [dict(T=300, V=1000, D=64, K=5), dict(T=257, V=2047, D=128, K=8), dict(T=200, V=777, D=256, K=16),
          dict(T=130, V=515, D=192, K=6)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"T{s['T']}_V{s['V']}_D{s['D']}")
@pytest.mark.parametrize("reduction", ["mean", "sum", "mean_elements"])
def test_weights_match_oracle(shape, reduction):
    p = W.draw(**shape, dtype="bf16", seed=31, ids="zipf", mask="random", mask_frac=0.1)
    w = weights_for(p, 1)
    got = call(p, to_device(p), reduction, weights=w)
    ref = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=RED[reduction], weights=w.astype(np.float64))
    assert got["n_valid"] == ref.n_valid and got["n_pairs"] == ref.n_pairs
    assert np.array_equal(got["row_counts"], ref.row_counts.astype(np.int32))
    assert abs(got["loss"] - ref.loss) <= LOSS_RTOL * abs(ref.loss), (got["loss"], ref.loss)
    dH = got["dH"].cpu().numpy()
    assert np.all(dH[(p.mask == 0) | (w == 0)] == 0.0)
    assert rel_fro(dH, ref.dH) <= GRAD_RTOL
    assert rel_fro(got["dE"].cpu().numpy(), ref.dE) <= GRAD_RTOL


def test_weights_with_one_signed_logits():
    # weighted loss (taken in the position-owned pass) whose linear half, from the
    # weighted column sums, is most of the loss
    p = W.draw(T=257, V=1500, D=128, K=6, dtype="bf16", seed=33, ids="zipf", mask="random", mask_frac=0.1)
    p.E_bits &= np.uint16(0x7FFF)
    p.E[:] = np.abs(p.E)
    p.H_bits &= np.uint16(0x7FFF)
    p.H[:] = np.abs(p.H)
    w = weights_for(p, 4)
    got = call(p, to_device(p), "sum", weights=w)
    ref = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=RED["sum"], weights=w.astype(np.float64))
    assert abs(got["loss"] - ref.loss) <= LOSS_RTOL * abs(ref.loss), (got["loss"], ref.loss)
    assert rel_fro(got["dH"].cpu().numpy(), ref.dH) <= GRAD_RTOL
    assert rel_fro(got["dE"].cpu().numpy(), ref.dE) <= GRAD_RTOL


@pytest.mark.parametrize("want", [("loss",), ("loss", "metrics"), ("dE",), ("dH",), ("loss", "dE")])
def test_weights_partial_outputs(want):
    p = W.draw(T=333, V=1500, D=64, K=4, dtype="bf16", seed=32, ids="zipf", mask="random", mask_frac=0.2)
    w = weights_for(p, 2)
    got = call(p, to_device(p), weights=w, want=tuple(x for x in want if x != "metrics"), metrics="metrics" in want)
    ref = O.forward_backward(p.H, p.E, p.targets, p.mask, weights=w.astype(np.float64))
    if "loss" in want:
        assert abs(got["loss"] - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    if "dE" in want:
        assert rel_fro(got["dE"].cpu().numpy(), ref.dE) <= GRAD_RTOL
    if "dH" in want:
        assert rel_fro(got["dH"].cpu().numpy(), ref.dH) <= GRAD_RTOL
    if "metrics" in want:
        refm = O.cut_metrics(p.H, p.E, p.targets, p.mask, weights=w)
        valid = (p.mask != 0) & (w != 0)
        assert np.all(got["metrics"][~valid] == 0)
        assert np.all(got["metrics"][valid].sum(axis=1) == p.V)
        assert np.mean(np.all(got["metrics"] == refm, axis=1)) > 0.99


def test_zero_one_weights_are_the_mask():
    p = W.draw(T=300, V=1200, D=64, K=6, dtype="bf16", seed=33, ids="zipf", mask="random", mask_frac=0.25)
    t = to_device(p)
    H, E, tg, m = t
    masked = call(p, t)
    weighted = call(p, (H, E, tg, None), weights=p.mask.astype(np.float32))
    # which positions and pairs contribute: bit for bit
    assert weighted["n_valid"] == masked["n_valid"] and weighted["n_pairs"] == masked["n_pairs"]
    assert np.array_equal(weighted["row_counts"], masked["row_counts"])
    # the values: the same problem, within the tolerance (the weighted path sums the loss in the other pass)
    ref = O.forward_backward(p.H, p.E, p.targets, p.mask)
    assert abs(weighted["loss"] - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert abs(weighted["loss"] - masked["loss"]) <= LOSS_RTOL * abs(ref.loss)
    assert rel_fro(weighted["dE"].cpu().numpy(), ref.dE) <= GRAD_RTOL
    assert rel_fro(weighted["dH"].cpu().numpy(), ref.dH) <= GRAD_RTOL
    assert np.all(weighted["dH"].cpu().numpy()[p.mask == 0] == 0.0)


@pytest.mark.parametrize("weighted", [False, True])
def test_bf16_outputs_are_the_rounded_fp32_outputs(weighted):
    p = W.draw(T=300, V=1000, D=64, K=5, dtype="bf16", seed=34, ids="zipf", mask="random", mask_frac=0.1)
    t = to_device(p)
    w = weights_for(p, 3) if weighted else None
    a = call(p, t, weights=w)
    b = call(p, t, weights=w, grad_dtype=B.GRAD_BF16)
    assert b["dH"].dtype == torch.bfloat16 and b["dE"].dtype == torch.bfloat16
    assert a["loss"] == b["loss"]
    assert torch.equal(a["dH"].to(torch.bfloat16), b["dH"])
    assert torch.equal(a["dE"].to(torch.bfloat16), b["dE"])


@pytest.mark.parametrize("grad_dtype", [B.GRAD_F32, B.GRAD_BF16])
def test_accumulate(grad_dtype):
    p = W.draw(T=257, V=2047, D=128, K=8, dtype="bf16", seed=35, ids="zipf", mask="random", mask_frac=0.1)
    t = to_device(p)
    fresh = call(p, t)                                 # fp32, overwritten
    g = torch.Generator(device="cuda").manual_seed(7)
    dt = torch.bfloat16 if grad_dtype == B.GRAD_BF16 else torch.float32
    init = (torch.randn((p.T, p.D), generator=g, device="cuda").to(dt),
            torch.randn((p.V, p.D), generator=g, device="cuda").to(dt))
    acc = call(p, t, grad_dtype=grad_dtype, accumulate=B.ACCUMULATE_DH | B.ACCUMULATE_DE, init=init)
    expect_dH = (init[0].float() + fresh["dH"]).to(dt)
    expect_dE = (init[1].float() + fresh["dE"]).to(dt)
    assert torch.equal(acc["dH"], expect_dH)           # masked rows keep their value
    assert torch.equal(acc["dE"], expect_dE)
    only_dE = call(p, t, grad_dtype=grad_dtype, accumulate=B.ACCUMULATE_DE, init=init)
    assert torch.equal(only_dE["dH"], fresh["dH"].to(dt))
    assert torch.equal(only_dE["dE"], expect_dE)


@pytest.mark.parametrize("reduction", ["mean", "mean_elements"])
@pytest.mark.parametrize("weighted", [False, True])
def test_vocabulary_shards(reduction, weighted):
    p = W.draw(T=300, V=2000, D=64, K=8, dtype="bf16", seed=36, ids="zipf", mask="random", mask_frac=0.1)
    t = to_device(p)
    H, E, tg, m = t
    w = weights_for(p, 4) if weighted else None
    full = call(p, t, reduction, weights=w, metrics=True)
    ref = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=RED[reduction],
                             weights=None if w is None else w.astype(np.float64))
    cuts = [0, 640, 641, 1400, p.V]                    # tile-aligned and ragged shard edges
    loss, dH, dE, met = 0.0, torch.zeros_like(full["dH"]), [], np.zeros((p.T, 4), dtype=np.int64)
    for v0, v1 in zip(cuts[:-1], cuts[1:]):
        r = call(p, t, reduction, weights=w, metrics=True, vocab_offset=v0, V_total=p.V, E=E[v0:v1].contiguous())
        assert r["n_valid"] == full["n_valid"]
        loss += r["loss"]
        dH += r["dH"]
        dE.append(r["dE"])
        met += r["metrics"]
    assert abs(loss - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert rel_fro(dH.cpu().numpy(), ref.dH) <= GRAD_RTOL
    assert rel_fro(torch.cat(dE).cpu().numpy(), ref.dE) <= GRAD_RTOL
    assert np.array_equal(met, full["metrics"])         # the same logits decide, shard by shard
    assert n_pairs_sum_ok(p, cuts)


def n_pairs_sum_ok(p, cuts):
    tg = O.positive_sets(p.targets, p.mask, p.V)
    total = sum(O.positive_sets(p.targets, p.mask, v1 - v0, vocab_offset=v0, V_total=p.V).n_pairs
                for v0, v1 in zip(cuts[:-1], cuts[1:]))
    return total == tg.n_pairs


def test_shard_id_range_errors():
    p = W.draw(T=64, V=500, D=64, K=3, dtype="bf16", seed=37, mask="none")
    t = to_device(p)
    H, E, tg, m = t
    p.targets[3, 1] = 900                              # inside V_total = 1000, another shard: fine
    tg_ok = torch.from_numpy(p.targets).cuda()
    ok = call(p, (H, E, tg_ok, m), vocab_offset=0, V_total=1000)
    assert ok["n_pairs"] == O.positive_sets(p.targets, p.mask, p.V, vocab_offset=0, V_total=1000).n_pairs
    p.targets[3, 1] = 1000                             # outside the whole vocabulary: a data error
    tg_bad = torch.from_numpy(p.targets).cuda()        # kept alive until the call has run
    prob = B.make_problem(H, E, tg_bad, m, "mean")
    opts = B.make_options(vocab_offset=0, V_total=1000)
    ws = torch.empty(B.cutbce_workspace_size_ex(prob, opts, B.OUT_LOSS), dtype=torch.uint8, device="cuda")
    loss = torch.empty((), dtype=torch.float64, device="cuda")
    B.cutbce_forward_backward_ex(prob, opts, None, loss, None, None, ws)
    assert B.cutbce_read_status(ws) == B.ERR_TARGET_RANGE
    del tg_bad


def test_fp32_path_options():
    p = W.draw_config("tiny_f32")
    w = weights_for(p, 5)
    got = call(p, to_device(p), weights=w, metrics=True)
    ref = O.forward_backward(p.H, p.E, p.targets, p.mask, weights=w.astype(np.float64))
    assert abs(got["loss"] - ref.loss) <= 1e-6 * abs(ref.loss)
    assert rel_fro(got["dH"].cpu().numpy(), ref.dH) <= 1e-5
    assert rel_fro(got["dE"].cpu().numpy(), ref.dE) <= 1e-5
    b = call(p, to_device(p), weights=w, grad_dtype=B.GRAD_BF16)
    assert torch.equal(got["dE"].to(torch.bfloat16), b["dE"])
