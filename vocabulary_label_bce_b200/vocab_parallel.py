"""Vocabulary-parallel fused BCE across GPUs ("Cut Binary Cross Entropy",
section III-C: the sharded backward with a vocabulary offset per shard and a sum
over the mesh).

Rank r of a group of size G owns the contiguous item rows [v0, v1) of E given
by shard_bounds (tile-aligned, balanced).  Every rank holds the same H, targets,
mask and weights.  Each rank runs the library on its shard with
cutbce_options.vocab_offset = v0 and V_total, which gives its share of the loss
sum and of dH (same normalisation on every rank, since the valid positions do
not depend on the shard) and its own rows of dE; one all-reduce (sum) of the
loss, of dH and, if asked, of the Cut Metrics counts then gives every rank the
unsharded loss, dH and metrics, while dE stays sharded.  The exchange is a
plain NCCL all-reduce over NVLink (torch.distributed); no operand of any kernel
is another GPU's memory.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

__all__ = ["shard_bounds", "vocab_parallel_forward_backward", "library_shard_compute"]

TILE = 128


def shard_bounds(V_total: int, world: int, rank: int, tile: int = TILE) -> tuple[int, int]:
    """Rows [v0, v1) of rank `rank`: the V_total items cut into `world` contiguous
    shards of whole 128-item tiles, as even as the tiles allow (earlier shards
    take the extra tiles); a shard may be empty only if there are fewer tiles
    than ranks."""
    if world < 1 or not 0 <= rank < world or V_total < 1:
        raise ValueError("bad shard request")
    tiles = -(-V_total // tile)
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(V_total, t0 * tile), min(V_total, t1 * tile)


def library_shard_compute(H, E_local, targets, mask, v0, V_total, reduction="mean", grad_loss=None, weights=None,
                          want_metrics=False):
    """This rank's share through the CUDA library: (loss, dH, dE_local, metrics or None)."""
    from . import binding as B
    prob = B.make_problem(H, E_local, targets, mask, reduction)
    met = torch.empty((H.shape[0], 4), dtype=torch.int32, device=H.device) if want_metrics else None
    opts = B.make_options(metrics=met, weights=weights, vocab_offset=v0, V_total=V_total)
    bits = B.OUT_LOSS | B.OUT_DH | B.OUT_DE | (B.OUT_METRICS if want_metrics else 0)
    ws = torch.empty(B.cutbce_workspace_size_ex(prob, opts, bits), dtype=torch.uint8, device=H.device)
    loss = torch.empty((), dtype=torch.float64, device=H.device)
    dH = torch.empty(H.shape, dtype=torch.float32, device=H.device)
    dE = torch.empty(E_local.shape, dtype=torch.float32, device=H.device)
    g = grad_loss.to(torch.float32).reshape(()) if grad_loss is not None else None
    B.cutbce_forward_backward_ex(prob, opts, g, loss, dH, dE, ws)
    status = B.cutbce_read_status(ws)
    if status != 0:
        raise B.CutBCEError(status, "vocab-parallel shard")
    return loss, dH, dE, met


def vocab_parallel_forward_backward(H, E_local, targets, mask, V_total: int, group=None, reduction="mean",
                                    grad_loss=None, weights=None, want_metrics=False,
                                    compute: Optional[Callable] = None):
    """Loss, dH (both summed over the group), this rank's dE rows and, if asked,
    the summed metrics.  E_local must be rows shard_bounds(V_total, G, r) of E."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    v0, v1 = shard_bounds(V_total, world, rank)
    if E_local.shape[0] != v1 - v0:
        raise ValueError(f"rank {rank} holds {E_local.shape[0]} rows, its shard is [{v0}, {v1})")
    if v1 > v0:
        fn = compute if compute is not None else library_shard_compute
        loss, dH, dE, met = fn(H, E_local, targets, mask, v0, V_total, reduction=reduction, grad_loss=grad_loss,
                               weights=weights, want_metrics=want_metrics)
    else:
        # more ranks than item tiles: this rank contributes nothing but still joins the exchange
        loss = torch.zeros((), dtype=torch.float64, device=H.device)
        dH = torch.zeros(H.shape, dtype=torch.float32, device=H.device)
        dE = torch.zeros((0, H.shape[1]), dtype=torch.float32, device=H.device)
        met = torch.zeros((H.shape[0], 4), dtype=torch.int32, device=H.device) if want_metrics else None
    # one exchange: the loss share and dH (and the integer counts) are summed over the ranks
    dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dH, op=dist.ReduceOp.SUM, group=group)
    if want_metrics:
        dist.all_reduce(met, op=dist.ReduceOp.SUM, group=group)
    return loss, dH, dE, met
