"""Float64 CPU oracle for the exact fused large-vocabulary BCE loss and its gradient.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg may import this module. The product path (the CUDA library and
its Python binding) never imports it, and it imports nothing from the product.

What it computes follows "Cut Binary Cross Entropy: Efficient Large-Vocabulary
Loss and Gradient Kernels for Sequential Recommendation" (Li, Ning, Hammad):

  * section III-A, Eq. (1): standard BCE of logit x and target y,
        l(x, y) = -y log s(x) - (1 - y) log(1 - s(x)),  s = logistic sigmoid;
  * section III-A, Eq. (2): the same value in the stable form
        l(x, y) = max(x, 0) + log(1 + exp(-|x|)) - y x = l(x, 0) - y x;
  * section III-A, Eq. (3): the loss of one position sums Eq. (2) over the whole
    vocabulary (with a 1/V factor);
  * section III-B, Eq. (4): dl/dx = s(x) - y, so with G = s(X) - Y,
        grad_A = G E  and  grad_E = G^T A,
    rows of A (here H) being the B*N flattened positions; averaging over the
    positions adds 1/(BN), padding positions excluded.

The logits X = A E^T are formed here chunk by chunk over the vocabulary (the
"vocabulary chunking" idea of section III-A), densely, in float64, with a
dense multi-hot Y inside the element loss (the Eq. (1)/(2) form), so that this
file is a plain restatement and shares no arithmetic with the GPU design.

Readings where the paper is silent:
  * normalisation: MEAN_VALID_POSITIONS (default) divides the summed loss by the
    number of valid positions; SUM does not divide; MEAN_ELEMENTS divides by
    n_valid * V (Eq. (3)'s 1/V times section III-B's 1/BN);
  * duplicate ids in a row count once (Y is multi-hot, y in {0, 1});
  * -1 marks an empty slot; an id < -1 or >= V in a valid row is an error;
    id 0 is an ordinary item;
  * a masked row adds no loss, gets a zero dH row and adds nothing to dE; its
    ids are ignored entirely (not even range-checked);
  * the per-position `weights` of the paper's API multiply the position's loss
    row and its row of G; a zero weight makes the position padding (excluded
    from the mean, like a masked one), so {0, 1} weights are the mask;
  * the upstream gradient is one scalar g (default 1) multiplying dH and dE;
  * with no valid position the loss and both gradients are 0.

Every function here is pinned by tests/test_oracle_pins.py against identities,
closed forms, finite differences, torch's own BCE-with-logits, brute-force
enumeration on tiny inputs and scikit-learn's classification metrics.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

MEAN_VALID_POSITIONS = 0
SUM = 1
MEAN_ELEMENTS = 2

LN2 = float(np.log(2.0))


class TargetRangeError(ValueError):
    """An id < -1 or >= V sits in a valid row."""


@dataclasses.dataclass
class Targets:
    """The positive sets P_t and the validity of each position (section III-B, sparse ids)."""
    valid: np.ndarray            # bool [T]
    sets: list                   # per row: sorted int64 array of distinct ids (empty if masked)

    @property
    def n_valid(self) -> int:
        return int(self.valid.sum())

    @property
    def row_counts(self) -> np.ndarray:
        return np.array([len(s) for s in self.sets], dtype=np.int64)

    @property
    def n_pairs(self) -> int:
        return int(self.row_counts.sum())


def positive_sets(targets: np.ndarray, mask: Optional[np.ndarray], V: int,
                  weights: Optional[np.ndarray] = None, vocab_offset: int = 0,
                  V_total: Optional[int] = None) -> Targets:
    """Apply the mask, the weights and the id rules: P_t = set of ids >= 0 in a valid row.

    A position is valid iff its mask entry is nonzero and its weight (if given) is
    nonzero.  With a vocabulary shard (vocab_offset, V_total), ids are global: an
    id outside [-1, V_total) is an error, an id outside [vocab_offset,
    vocab_offset + V) is not in this shard and is dropped, and the kept ids are
    returned shard-local (id - vocab_offset)."""
    targets = np.asarray(targets)
    T = targets.shape[0]
    Vt = V if V_total is None else int(V_total)
    valid = np.ones(T, dtype=bool) if mask is None else (np.asarray(mask) != 0)
    if weights is not None:
        valid = valid & (np.asarray(weights, dtype=np.float64) != 0.0)
    sets = []
    for t in range(T):
        if not valid[t]:
            sets.append(np.zeros(0, dtype=np.int64))
            continue
        row = targets[t].astype(np.int64)
        if np.any(row < -1) or np.any(row >= Vt):
            raise TargetRangeError(f"row {t}: id outside [-1, {Vt})")
        local = row[(row >= vocab_offset) & (row < vocab_offset + V)] - vocab_offset
        sets.append(np.unique(local))
    return Targets(valid=valid, sets=sets)


def sigmoid(x: np.ndarray) -> np.ndarray:
    """Logistic sigmoid, two-branch form that never overflows."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def bce_eq1(x: np.ndarray, y: np.ndarray) -> np.ndarray:
    """Eq. (1): -y log s(x) - (1-y) log(1 - s(x)), evaluated literally (moderate |x| only)."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    p = 1.0 / (1.0 + np.exp(-x))
    return -y * np.log(p) - (1.0 - y) * np.log(1.0 - p)


def bce_eq2(x: np.ndarray, y: np.ndarray) -> np.ndarray:
    """Eq. (2): max(x, 0) + log(1 + exp(-|x|)) - y x."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x))) - y * x


def scale_factor(reduction: int, n_valid: int, V: int) -> float:
    """Normalisation s applied to the summed loss and to both gradients."""
    if n_valid == 0:
        return 0.0
    if reduction == MEAN_VALID_POSITIONS:
        return 1.0 / n_valid
    if reduction == SUM:
        return 1.0
    if reduction == MEAN_ELEMENTS:
        return 1.0 / (float(n_valid) * float(V))
    raise ValueError(f"unknown reduction {reduction}")


def _multi_hot(sets_valid: Sequence[np.ndarray], c0: int, c1: int) -> np.ndarray:
    Y = np.zeros((len(sets_valid), c1 - c0), dtype=np.float64)
    for r, ids in enumerate(sets_valid):
        sel = ids[(ids >= c0) & (ids < c1)]
        Y[r, sel - c0] = 1.0
    return Y


@dataclasses.dataclass
class Result:
    loss: float
    dH: Optional[np.ndarray]
    dE: Optional[np.ndarray]
    sum_loss: float              # unnormalised sum of Eq. (2) over valid rows and all items
    n_valid: int
    n_pairs: int
    row_counts: np.ndarray


def forward_backward(H: np.ndarray, E: np.ndarray, targets: np.ndarray,
                     mask: Optional[np.ndarray] = None, reduction: int = MEAN_VALID_POSITIONS,
                     grad_loss: float = 1.0, chunk: int = 8192, want_grad: bool = True,
                     weights: Optional[np.ndarray] = None, vocab_offset: int = 0,
                     V_total: Optional[int] = None) -> Result:
    """Loss and gradients of the fused BCE, computed densely chunk by chunk over V.

    H [T, D] and E [V, D] are taken as given (the exact input values, widened to
    float64); targets [T, K] int ids with -1 empty; mask [T] (nonzero = valid).

    weights [T] (the per-position weights of the paper's API, section III-C
    Listing 1): position t's loss row and its row of G are multiplied by w_t, so
    loss = s sum_t w_t sum_v l(x_tv, y_tv), G = diag(w) (sigmoid(X) - Y); a
    position with w_t = 0 is padding (not counted in the mean).

    vocab_offset, V_total: E holds items [vocab_offset, vocab_offset + V) of a
    vocabulary of V_total items (one shard of a vocabulary-parallel split): the
    result is this shard's share of the loss sum and of dH (the shares of all
    shards add up to the unsharded result) and the shard's rows of dE.  The
    MEAN_ELEMENTS normalisation uses V_total.
    """
    H64 = np.asarray(H, dtype=np.float64)
    E64 = np.asarray(E, dtype=np.float64)
    T, D = H64.shape
    V = E64.shape[0]
    Vt = V if V_total is None else int(V_total)
    tg = positive_sets(targets, mask, V, weights, vocab_offset, Vt)
    rows = np.nonzero(tg.valid)[0]
    Hv = H64[rows]
    sets_v = [tg.sets[t] for t in rows]
    w = np.ones(len(rows)) if weights is None else np.asarray(weights, dtype=np.float64)[rows]

    total = 0.0
    dHv = np.zeros_like(Hv) if want_grad else None
    dE = np.zeros((V, D), dtype=np.float64) if want_grad else None
    if len(rows):
        for c0 in range(0, V, chunk):
            c1 = min(V, c0 + chunk)
            Ec = E64[c0:c1]
            Z = Hv @ Ec.T                                  # chunk logits, then discarded
            Y = _multi_hot(sets_v, c0, c1)
            total += float((w[:, None] * bce_eq2(Z, Y)).sum())   # Eq. (2), summed as in Eq. (3)
            if want_grad:
                G = w[:, None] * (sigmoid(Z) - Y)          # Eq. (4), row t scaled by w_t
                dHv += G @ Ec
                dE[c0:c1] = G.T @ Hv
    s = scale_factor(reduction, len(rows), Vt)
    dH = None
    if want_grad:
        dH = np.zeros((T, D), dtype=np.float64)
        dH[rows] = grad_loss * s * dHv
        dE *= grad_loss * s
    return Result(loss=s * total, dH=dH, dE=dE, sum_loss=total, n_valid=len(rows),
                  n_pairs=tg.n_pairs, row_counts=tg.row_counts)


def dE_rows(H: np.ndarray, E: np.ndarray, targets: np.ndarray, mask: Optional[np.ndarray],
            items: Sequence[int], reduction: int = MEAN_VALID_POSITIONS,
            grad_loss: float = 1.0) -> np.ndarray:
    """Selected rows of grad_E (Eq. (4)), each from its own logit column X[:, v]."""
    H64 = np.asarray(H, dtype=np.float64)
    V = E.shape[0]
    tg = positive_sets(targets, mask, V)
    rows = np.nonzero(tg.valid)[0]
    Hv = H64[rows]
    s = scale_factor(reduction, len(rows), V)
    # the valid rows (indices into rows) that hold each positive item
    holders: dict = {}
    for r, t in enumerate(rows):
        for v in tg.sets[t].tolist():
            holders.setdefault(v, []).append(r)
    out = np.zeros((len(items), H64.shape[1]), dtype=np.float64)
    for i, v in enumerate(items):
        z = Hv @ np.asarray(E[v], dtype=np.float64)
        y = np.zeros(len(rows), dtype=np.float64)
        y[holders.get(int(v), [])] = 1.0
        out[i] = grad_loss * s * ((sigmoid(z) - y) @ Hv)
    return out


def dH_rows(H: np.ndarray, E: np.ndarray, targets: np.ndarray, mask: Optional[np.ndarray],
            positions: Sequence[int], reduction: int = MEAN_VALID_POSITIONS,
            grad_loss: float = 1.0, chunk: int = 1 << 18) -> np.ndarray:
    """Selected rows of grad_A = grad_H (Eq. (4)), each from its own logit row X[t, :].

    The vocabulary is walked chunk by chunk; within a chunk every selected row's
    logits, sigmoid minus targets and contribution are formed densely."""
    V = E.shape[0]
    tg = positive_sets(targets, mask, V)
    s = scale_factor(reduction, tg.n_valid, V)
    pos = [t for t in positions if tg.valid[t]]
    Hs = np.asarray(H, dtype=np.float64)[pos]
    acc = np.zeros((len(pos), H.shape[1]), dtype=np.float64)
    for c0 in range(0, V, chunk):
        c1 = min(V, c0 + chunk)
        Ec = np.asarray(E[c0:c1], dtype=np.float64)
        Z = Hs @ Ec.T
        Y = _multi_hot([tg.sets[t] for t in pos], c0, c1)
        acc += (sigmoid(Z) - Y) @ Ec
    out = np.zeros((len(positions), H.shape[1]), dtype=np.float64)
    k = 0
    for i, t in enumerate(positions):
        if tg.valid[t]:
            out[i] = grad_loss * s * acc[k]
            k += 1
    return out


def loss_sum_slice(H: np.ndarray, E: np.ndarray, targets: np.ndarray, mask: Optional[np.ndarray],
                   v0: int, v1: int, chunk: int = 8192) -> float:
    """Unnormalised Eq. (2) sum restricted to the items [v0, v1) (all valid rows)."""
    V = E.shape[0]
    tg = positive_sets(targets, mask, V)
    rows = np.nonzero(tg.valid)[0]
    Hv = np.asarray(H, dtype=np.float64)[rows]
    sets_v = [tg.sets[t] for t in rows]
    total = 0.0
    for c0 in range(v0, v1, chunk):
        c1 = min(v1, c0 + chunk)
        Z = Hv @ np.asarray(E[c0:c1], dtype=np.float64).T
        total += float(bce_eq2(Z, _multi_hot(sets_v, c0, c1)).sum())
    return total


# ---------------------------------------------------------------- Cut Metrics (section III-D)
# Confusion counts per position over the whole vocabulary, computed from the
# logits without keeping them.  The pages give the four counts of shape [B, N]
# and say accuracy, precision, recall and F_beta follow from them; they do not
# state the decision threshold.  Reading: item v is predicted positive for
# position t iff sigmoid(x_tv) > 1/2, i.e. x_tv > 0 (a logit of exactly 0 is a
# predicted negative).  A masked position has all four counts 0.

def cut_metrics(H: np.ndarray, E: np.ndarray, targets: np.ndarray, mask: Optional[np.ndarray] = None,
                chunk: int = 8192, weights: Optional[np.ndarray] = None, vocab_offset: int = 0,
                V_total: Optional[int] = None) -> np.ndarray:
    """int64 [T, 4]: (TP, FP, FN, TN) of each position, from the dense logits chunk by chunk.

    The counts are not weighted; a position with weight 0 is padding (all zero).
    On a vocabulary shard the counts cover the shard's items only (the counts of
    all shards add up to the unsharded counts)."""
    H64 = np.asarray(H, dtype=np.float64)
    V = E.shape[0]
    tg = positive_sets(targets, mask, V, weights, vocab_offset, V if V_total is None else V_total)
    rows = np.nonzero(tg.valid)[0]
    Hv = H64[rows]
    sets_v = [tg.sets[t] for t in rows]
    counts = np.zeros((H64.shape[0], 4), dtype=np.int64)
    if len(rows) == 0:
        return counts
    acc = np.zeros((len(rows), 4), dtype=np.int64)
    for c0 in range(0, V, chunk):
        c1 = min(V, c0 + chunk)
        Z = Hv @ np.asarray(E[c0:c1], dtype=np.float64).T
        pred = Z > 0.0
        y = _multi_hot(sets_v, c0, c1) > 0.5
        acc[:, 0] += np.sum(pred & y, axis=1)
        acc[:, 1] += np.sum(pred & ~y, axis=1)
        acc[:, 2] += np.sum(~pred & y, axis=1)
        acc[:, 3] += np.sum(~pred & ~y, axis=1)
    counts[rows] = acc
    return counts


def metrics_from_counts(counts: np.ndarray, beta: float = 1.0) -> dict:
    """Binary accuracy, precision, recall and F_beta of the counts summed over positions
    (a ratio with a zero denominator is 0)."""
    tp, fp, fn, tn = (float(x) for x in np.asarray(counts, dtype=np.int64).reshape(-1, 4).sum(axis=0))
    total = tp + fp + fn + tn
    precision = tp / (tp + fp) if tp + fp > 0 else 0.0
    recall = tp / (tp + fn) if tp + fn > 0 else 0.0
    b2 = beta * beta
    denom = b2 * precision + recall
    fbeta = (1.0 + b2) * precision * recall / denom if denom > 0 else 0.0
    return {"accuracy": (tp + tn) / total if total > 0 else 0.0, "precision": precision, "recall": recall,
            "fbeta": fbeta}


# ---------------------------------------------------------------- full-vocabulary top-k and Hit@k (section III-E)
# Evaluation: a query (the hidden state of a sequence's last non-pad position)
# is scored against every item, x_v = q . e_v; the k highest scores rank the
# items; a query is a hit if at least one of its held-out target ids is among
# them (Hit@8 in the pages: k = 8, 8 held-out items).  Reading where the pages
# are silent: items are ranked by descending score, equal scores by ascending
# id; -1 marks an empty target slot; a query with no target is not a hit.

def topk(Q: np.ndarray, E: np.ndarray, k: int, chunk: int = 65536):
    """(ids int64 [B, k], scores float64 [B, k]): the k best items of each query."""
    Q64 = np.asarray(Q, dtype=np.float64)
    B, V = Q64.shape[0], E.shape[0]
    k = min(k, V)
    best_s = np.full((B, 0), -np.inf)
    best_i = np.zeros((B, 0), dtype=np.int64)
    for c0 in range(0, V, chunk):
        c1 = min(V, c0 + chunk)
        S = Q64 @ np.asarray(E[c0:c1], dtype=np.float64).T
        cand_s = np.concatenate([best_s, S], axis=1)
        cand_i = np.concatenate([best_i, np.broadcast_to(np.arange(c0, c1), S.shape)], axis=1)
        kk = min(k, cand_s.shape[1])                             # the first chunks may hold fewer than k
        keep_s = np.empty((B, kk))
        keep_i = np.empty((B, kk), dtype=np.int64)
        for b in range(B):
            order = np.lexsort((cand_i[b], -cand_s[b]))[:kk]     # score descending, then id ascending
            keep_s[b] = cand_s[b, order]
            keep_i[b] = cand_i[b, order]
        best_s, best_i = keep_s, keep_i
    return best_i, best_s


def hit_at_k(topk_ids: np.ndarray, targets: np.ndarray) -> np.ndarray:
    """int64 [B]: 1 if a target id (>= 0) of the query is among its top-k ids."""
    ids = np.asarray(topk_ids)
    tg = np.asarray(targets)
    return np.array([int(np.any(np.isin(tg[b][tg[b] >= 0], ids[b]))) for b in range(ids.shape[0])],
                    dtype=np.int64)
