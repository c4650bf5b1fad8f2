"""Vocabulary-parallel split on CPU: two gloo ranks, each computing its shard's
share with the oracle (the CUDA library needs a GPU), joined by the product's
partition and exchange code (vocabulary_label_bce_b200.vocab_parallel).  The
summed loss, dH and Cut Metrics and the gathered dE must equal the unsharded
oracle ("Cut Binary Cross Entropy", section III-C: per-shard vocabulary offset,
sum over the mesh)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from vocabulary_label_bce_b200.vocab_parallel import shard_bounds, vocab_parallel_forward_backward


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_shard_compute(H, E_local, targets, mask, v0, V_total, reduction="mean", grad_loss=None, weights=None,
                         want_metrics=False):
    from oracle import cutbce_oracle as O
    red = {"mean": O.MEAN_VALID_POSITIONS, "sum": O.SUM, "mean_elements": O.MEAN_ELEMENTS}[reduction]
    w = None if weights is None else weights.numpy().astype(np.float64)
    r = O.forward_backward(H.numpy(), E_local.numpy(), targets.numpy(), mask.numpy(), reduction=red,
                           grad_loss=1.0 if grad_loss is None else float(grad_loss), weights=w, vocab_offset=v0,
                           V_total=V_total)
    met = None
    if want_metrics:
        met = torch.from_numpy(O.cut_metrics(H.numpy(), E_local.numpy(), targets.numpy(), mask.numpy(), weights=w,
                                             vocab_offset=v0, V_total=V_total))
    return (torch.tensor(r.loss, dtype=torch.float64), torch.from_numpy(r.dH), torch.from_numpy(r.dE), met)


def _problem():
    from vocabulary_label_bce_b200 import workloads as W
    p = W.draw(T=48, V=700, D=8, K=6, dtype="f32", seed=5, ids="zipf", mask="random", mask_frac=0.15)
    w = np.random.default_rng(6).uniform(0.5, 1.5, p.T).astype(np.float32)
    return p, w


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p, w = _problem()
        v0, v1 = shard_bounds(p.V, world, rank)
        H = torch.from_numpy(p.H)
        loss, dH, dE, met = vocab_parallel_forward_backward(
            H, torch.from_numpy(p.E[v0:v1]), torch.from_numpy(p.targets), torch.from_numpy(p.mask), p.V,
            reduction="mean", grad_loss=torch.tensor(0.5), weights=torch.from_numpy(w), want_metrics=True,
            compute=oracle_shard_compute)
        parts = [None] * world
        dist.all_gather_object(parts, dE.numpy())
        out[rank] = (float(loss), dH.numpy(), np.concatenate(parts), met.numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_equal_the_unsharded_oracle():
    from oracle import cutbce_oracle as O
    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    p, w = _problem()
    ref = O.forward_backward(p.H, p.E, p.targets, p.mask, grad_loss=0.5, weights=w.astype(np.float64))
    refm = O.cut_metrics(p.H, p.E, p.targets, p.mask, weights=w)
    for rank in range(world):
        loss, dH, dE, met = out[rank]
        assert loss == pytest.approx(ref.loss, rel=1e-12)
        assert np.allclose(dH, ref.dH, rtol=1e-12, atol=1e-15)
        assert np.allclose(dE, ref.dE, rtol=1e-12, atol=1e-15)
        assert np.array_equal(met, refm)


@pytest.mark.parametrize("V,world", [(876_000, 8), (1000, 3), (130, 2), (100, 4)])
def test_shard_bounds_partition(V, world):
    b = [shard_bounds(V, world, r) for r in range(world)]
    assert b[0][0] == 0 and b[-1][1] == V
    for (a0, a1), (c0, c1) in zip(b[:-1], b[1:]):
        assert a1 == c0 and a0 <= a1
    assert all(v0 % 128 == 0 or v0 == V for v0, _ in b)         # whole tiles; an empty shard sits at V
    tiles = [-(-(v1 - v0) // 128) for v0, v1 in b]
    assert max(tiles) - min(tiles) <= 1
