"""Helpers shared by the GPU parity tests: move a drawn problem to the device,
call the library through its C ABI, and compare with the float64 oracle."""
import numpy as np
import torch

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import binding as B

LOSS_RTOL = 1e-5        # relative error of the loss
GRAD_RTOL = 2e-3        # relative Frobenius error of dH and dE
RED = {"mean": O.MEAN_VALID_POSITIONS, "sum": O.SUM, "mean_elements": O.MEAN_ELEMENTS}


def to_device(p, device="cuda"):
    if p.dtype == "bf16":
        H = torch.from_numpy(p.H_bits.view(np.int16)).view(torch.bfloat16).to(device)
        E = torch.from_numpy(p.E_bits.view(np.int16)).view(torch.bfloat16).to(device)
    else:
        H = torch.from_numpy(p.H).to(device)
        E = torch.from_numpy(p.E).to(device)
    tg = torch.from_numpy(p.targets).to(device)
    m = torch.from_numpy(p.mask).to(device)
    return H, E, tg, m


def run_gpu(p, reduction="mean", grad_loss=None, entry="fused", tensors=None, use_mask=True):
    H, E, tg, m = tensors if tensors is not None else to_device(p)
    prob = B.make_problem(H, E, tg, m if use_mask else None, reduction)
    ws = torch.empty(B.cutbce_workspace_size(prob), dtype=torch.uint8, device=H.device)
    g = torch.tensor(grad_loss, dtype=torch.float32, device=H.device) if grad_loss is not None else None
    loss = torch.full((), float("nan"), dtype=torch.float64, device=H.device)
    dH = torch.full((p.T, p.D), float("nan"), dtype=torch.float32, device=H.device)
    dE = torch.full((p.V, p.D), float("nan"), dtype=torch.float32, device=H.device)
    if entry == "fused":
        B.cutbce_forward_backward(prob, g, loss, dH, dE, ws)
    elif entry == "forward":
        B.cutbce_forward(prob, ws, loss)
        dH = dE = None
    elif entry == "backward":
        B.cutbce_backward(prob, g, dH, dE, ws)
        loss = None
    status = B.cutbce_read_status(ws)
    torch.cuda.synchronize()
    out = {"status": status, "prob": prob, "ws": ws,
           "loss": None if loss is None else float(loss.item()),
           "dH": None if dH is None else dH.cpu().numpy().astype(np.float64),
           "dE": None if dE is None else dE.cpu().numpy().astype(np.float64)}
    return out


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def check_against_oracle(p, got, reduction="mean", grad_loss=1.0, loss_rtol=LOSS_RTOL, grad_rtol=GRAD_RTOL,
                         chunk=8192):
    ref = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=RED[reduction],
                             grad_loss=1.0 if grad_loss is None else grad_loss, chunk=chunk)
    assert got["status"] == 0, B.cutbce_status_string(got["status"])
    report = {}
    if got["loss"] is not None:
        err = abs(got["loss"] - ref.loss) / max(abs(ref.loss), 1e-300) if ref.loss != 0 else abs(got["loss"])
        report["loss_rel"] = err
        assert err <= loss_rtol, (got["loss"], ref.loss, err)
    if got["dH"] is not None:
        report["dH_rel"] = rel_fro(got["dH"], ref.dH)
        assert np.all(got["dH"][p.mask == 0] == 0.0), "masked rows of dH must be exactly 0"
        assert report["dH_rel"] <= grad_rtol, report
    if got["dE"] is not None:
        report["dE_rel"] = rel_fro(got["dE"], ref.dE)
        assert report["dE_rel"] <= grad_rtol, report
    # which terms contribute: integer side results are bit-exact
    rc = torch.empty(p.T, dtype=torch.int32)
    nv, npairs = B.cutbce_read_counts(got["prob"], got["ws"], rc)
    assert nv == ref.n_valid and npairs == ref.n_pairs
    assert np.array_equal(rc.numpy(), ref.row_counts.astype(np.int32))
    return ref, report
