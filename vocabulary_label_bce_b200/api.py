"""torch-facing calls of the fused large-vocabulary BCE (device tensors in, device tensors out).

PyTorch supplies device memory and the current stream; all arithmetic runs in
libcutbce's kernels (see include/cutbce.h).
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B

__all__ = ["forward", "backward", "forward_backward", "cut_bce", "Workspace"]


class Workspace:
    """Caches one device workspace per (device, size); grows on demand."""

    def __init__(self):
        self._buf: dict[int, torch.Tensor] = {}

    def get(self, nbytes: int, device: torch.device) -> torch.Tensor:
        idx = device.index if device.index is not None else torch.cuda.current_device()
        buf = self._buf.get(idx)
        if buf is None or buf.numel() < nbytes:
            buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
            self._buf[idx] = buf
        return buf


_WS = Workspace()


def _mask_u8(mask: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if mask is None:
        return None
    return mask.to(torch.uint8).contiguous() if mask.dtype != torch.uint8 else mask.contiguous()


def _flat(H, targets, mask):
    # [B, N, D] activations and [B, N, L] ids are flattened to T = B*N rows
    if H.dim() == 3:
        H = H.reshape(-1, H.shape[-1])
    if targets.dim() == 3:
        targets = targets.reshape(-1, targets.shape[-1])
    if mask is not None and mask.dim() == 2:
        mask = mask.reshape(-1)
    return H.contiguous(), targets.to(torch.int32).contiguous(), _mask_u8(mask)


def forward_backward(H: torch.Tensor, E: torch.Tensor, targets: torch.Tensor, mask: Optional[torch.Tensor] = None,
                     reduction: str = "mean", grad_loss: Optional[torch.Tensor] = None, want_loss: bool = True,
                     want_dH: bool = True, want_dE: bool = True, workspace: Optional[torch.Tensor] = None):
    """Loss (0-d float64) and gradients dH [T, D], dE [V, D] (float32); None for what was not asked."""
    H2, tg, m = _flat(H, targets, mask)
    E = E.contiguous()
    prob = B.make_problem(H2, E, tg, m, reduction)
    outs = (B.OUT_LOSS if want_loss else 0) | (B.OUT_DH if want_dH else 0) | (B.OUT_DE if want_dE else 0)
    ws = workspace if workspace is not None else _WS.get(B.cutbce_workspace_size_for(prob, outs), H2.device)
    loss = torch.empty((), dtype=torch.float64, device=H2.device) if want_loss else None
    dH = torch.empty(H2.shape, dtype=torch.float32, device=H2.device) if want_dH else None
    dE = torch.empty(E.shape, dtype=torch.float32, device=E.device) if want_dE else None
    g = grad_loss.to(torch.float32).reshape(()) if grad_loss is not None else None
    B.cutbce_forward_backward(prob, g, loss, dH, dE, ws)
    if dH is not None and H.dim() == 3:
        dH = dH.reshape(H.shape)
    return loss, dH, dE


def forward(H, E, targets, mask=None, reduction: str = "mean", workspace=None) -> torch.Tensor:
    H2, tg, m = _flat(H, targets, mask)
    E = E.contiguous()
    prob = B.make_problem(H2, E, tg, m, reduction)
    ws = workspace if workspace is not None else _WS.get(B.cutbce_workspace_size_for(prob, B.OUT_LOSS), H2.device)
    loss = torch.empty((), dtype=torch.float64, device=H2.device)
    B.cutbce_forward(prob, ws, loss)
    return loss


def backward(H, E, targets, mask=None, reduction: str = "mean", grad_loss=None, want_dH=True, want_dE=True,
             workspace=None):
    H2, tg, m = _flat(H, targets, mask)
    E = E.contiguous()
    prob = B.make_problem(H2, E, tg, m, reduction)
    outs = (B.OUT_DH if want_dH else 0) | (B.OUT_DE if want_dE else 0)
    ws = workspace if workspace is not None else _WS.get(B.cutbce_workspace_size_for(prob, outs), H2.device)
    dH = torch.empty(H2.shape, dtype=torch.float32, device=H2.device) if want_dH else None
    dE = torch.empty(E.shape, dtype=torch.float32, device=E.device) if want_dE else None
    g = grad_loss.to(torch.float32).reshape(()) if grad_loss is not None else None
    B.cutbce_backward(prob, g, dH, dE, ws)
    if dH is not None and H.dim() == 3:
        dH = dH.reshape(H.shape)
    return dH, dE


class _CutBCE(torch.autograd.Function):
    """Custom VJP in the paper's sense (section III-B): the forward keeps only H, E and
    the sparse ids; the backward recomputes every logit tile on chip."""

    @staticmethod
    def forward(ctx, H, E, targets, mask, reduction):
        ctx.save_for_backward(H, E, targets, mask if mask is not None else torch.empty(0))
        ctx.has_mask = mask is not None
        ctx.reduction = reduction
        return forward(H.detach(), E.detach(), targets, mask, reduction).to(torch.float32)

    @staticmethod
    def backward(ctx, grad):
        H, E, targets, mask = ctx.saved_tensors
        m = mask if ctx.has_mask else None
        dH, dE = backward(H.detach(), E.detach(), targets, m, ctx.reduction, grad_loss=grad,
                          want_dH=ctx.needs_input_grad[0], want_dE=ctx.needs_input_grad[1])
        dH = dH.to(H.dtype) if dH is not None else None
        dE = dE.to(E.dtype) if dE is not None else None
        return dH, dE, None, None, None


def cut_bce(H, E, targets, mask=None, reduction: str = "mean") -> torch.Tensor:
    """Differentiable fused BCE loss over the full vocabulary (autograd-aware)."""
    return _CutBCE.apply(H, E, targets, mask, reduction)
