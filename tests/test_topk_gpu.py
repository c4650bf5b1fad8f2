"""Full-vocabulary top-k and Hit@k on the GPU ("Cut Binary Cross Entropy",
section III-E) against the float64 oracle.

The kernel ranks by its fp32 accumulation of the bf16 products; the oracle by
the exact float64 score.  Their rankings can differ only among items whose
exact scores lie within the accumulation error of each other, so with
tau = 2^-16 * max_v sum_d |q_d e_vd| per query: every GPU score is within tau
of the exact score of its item; the GPU list is sorted by (its score
descending, id ascending); every item whose exact score beats the oracle's
k-th by more than 2 tau is chosen, and no chosen item trails it by more than
2 tau.  Where the exact scores around the list are more than 2 tau apart, the
ids must match the oracle's in order.  Exactly equal scores (duplicate item
rows) must come out by ascending id."""
import numpy as np
import pytest
import torch

from oracle import cutbce_oracle as O
from vocabulary_label_bce_b200 import binding as B
from vocabulary_label_bce_b200 import workloads as W

pytestmark = pytest.mark.gpu

TAU_REL = 2.0 ** -16


def bf16_tensor(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def check(Qf, Ef, k, ids, scores):
    Q64 = Qf.astype(np.float64)
    Bn, V = Q64.shape[0], Ef.shape[0]
    ref_i, ref_s = O.topk(Qf, Ef, k)
    tau = TAU_REL * np.max(np.abs(Q64) @ np.abs(Ef.astype(np.float64)).T, axis=1)
    exact_rows = 0
    for b in range(Bn):
        gi, gs = ids[b], scores[b]
        assert len(set(gi.tolist())) == k and np.all((gi >= 0) & (gi < V))
        ex = Q64[b] @ Ef[gi].astype(np.float64).T
        assert np.all(np.abs(gs - ex) <= tau[b]), b
        for j in range(k - 1):                       # the kernel's own order
            assert gs[j] > gs[j + 1] or (gs[j] == gs[j + 1] and gi[j] < gi[j + 1]), (b, j)
        kth = ref_s[b, -1]
        assert np.all(ex >= kth - 2 * tau[b]), b
        must = ref_i[b][ref_s[b] > kth + 2 * tau[b]]
        assert np.all(np.isin(must, gi)), b
        # no near-ties around the list: the ids must match in order
        allv = Q64[b] @ Ef.astype(np.float64).T
        near_boundary = np.sum(np.abs(allv - kth) <= 2 * tau[b]) > 1
        gaps = np.diff(ref_s[b])
        if not near_boundary and np.all(np.abs(gaps) > 2 * tau[b]):
            assert np.array_equal(gi, ref_i[b]), b
            exact_rows += 1
    return exact_rows


CASES = [
    dict(B=64, V=1000, D=64, k=8),
    dict(B=200, V=2047, D=128, k=16),       # two query tiles, a ragged item tile
    dict(B=1, V=777, D=256, k=5),           # 64-row item tiles
    dict(B=129, V=3000, D=40, k=1),         # D padded to 64
    dict(B=70, V=515, D=192, k=8),
    dict(B=33, V=6, D=64, k=8),             # fewer items than k
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}_V{c['V']}_D{c['D']}_k{c['k']}")
def test_topk_matches_oracle(case):
    rng = np.random.default_rng(41)
    Qb = W.to_bf16_bits(rng.standard_normal((case["B"], case["D"])).astype(np.float32))
    Eb = W.to_bf16_bits((rng.standard_normal((case["V"], case["D"])) / np.sqrt(case["D"])).astype(np.float32))
    Qf, Ef = W.bf16_bits_to_f32(Qb), W.bf16_bits_to_f32(Eb)
    ids, scores = B.cutbce_topk(bf16_tensor(Qb), bf16_tensor(Eb), case["k"])
    torch.cuda.synchronize()
    ids, scores = ids.cpu().numpy(), scores.cpu().numpy()
    k = case["k"]
    if case["V"] < k:
        ref_i, _ = O.topk(Qf, Ef, k)
        assert np.all(ids[:, case["V"]:] == -1)
        assert np.array_equal(np.sort(ids[:, :case["V"]], axis=1), np.sort(ref_i, axis=1))
        return
    n = check(Qf, Ef, k, ids, scores)
    print(case, "rows compared in exact order:", n)
    assert n >= case["B"] // 2


def test_equal_scores_come_out_by_id():
    rng = np.random.default_rng(42)
    base = rng.standard_normal((50, 64)).astype(np.float32) / 8
    Ef = np.repeat(base, 3, axis=0)               # items 3i, 3i+1, 3i+2 are identical
    Qf = rng.standard_normal((10, 64)).astype(np.float32)
    Qb, Eb = W.to_bf16_bits(Qf), W.to_bf16_bits(Ef)
    ids, scores = B.cutbce_topk(bf16_tensor(Qb), bf16_tensor(Eb), 9)
    ids = ids.cpu().numpy()
    for b in range(10):
        groups = ids[b].reshape(3, 3)
        for g in groups:                          # each best row appears as its three copies, ids ascending
            assert g[0] % 3 == 0 and g.tolist() == [g[0], g[0] + 1, g[0] + 2], ids[b]


def test_hit_at_8_sasrec_shape():
    # evaluation of the SASRec-style head: one query per sequence (its last valid
    # position), V = 876,000 items, 8 held-out Zipf(1.05) target ids per query
    p = W.draw_config("sasrec_876k")
    last = np.array([b * p.N + np.nonzero(p.mask[b * p.N:(b + 1) * p.N])[0][-1] for b in range(p.B)])
    Qb = np.ascontiguousarray(p.H_bits[last])
    Qf = p.H[last]
    rng = np.random.default_rng(43)
    cdf = np.cumsum(np.arange(1, p.V + 1, dtype=np.float64) ** -1.05)
    targets = np.minimum(np.searchsorted(cdf / cdf[-1], rng.random((p.B, 8))), p.V - 1).astype(np.int32)
    # make some queries hit: plant the query's own best item as a target
    E = bf16_tensor(p.E_bits)
    ids, scores = B.cutbce_topk(bf16_tensor(Qb), E, 8)
    targets[::3, 0] = ids.cpu().numpy()[::3, 0]
    hits = B.cutbce_hit_at_k(ids, torch.from_numpy(targets).cuda())
    ids_np, scores_np = ids.cpu().numpy(), scores.cpu().numpy()
    n = check(Qf, p.E, 8, ids_np, scores_np)
    assert n >= p.B // 2
    assert np.array_equal(hits.cpu().numpy(), O.hit_at_k(ids_np, targets))
    assert hits.cpu().numpy()[::3].min() == 1
