"""Write fullv_loss.json: the float64 oracle's summed loss over the whole vocabulary
for the three large workloads (SASRec-style head, wide embedding, extreme catalog).

Calls only oracle/ and the seeded input generator.  The sum of Eq. (2) of "Cut
Binary Cross Entropy" (section III-A) over every valid position and every item
is additive over the items, so the vocabulary is cut into contiguous slices,
each slice's sum is taken by oracle.loss_sum_slice on its own thread (numpy
releases the interpreter lock inside its array kernels), and the slice sums are
added in slice order.

    python tests/golden/make_fullv_loss.py [workload ...]
"""
import json
import os
import sys
import time
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import cutbce_oracle as O  # noqa: E402
from vocabulary_label_bce_b200 import workloads as W  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "fullv_loss.json")
WORKLOADS = ["sasrec_876k", "wide_d256", "extreme_10m"]
SEED = 0
SLICES = 256          # vocabulary slices (work items for the thread pool)
CHUNK = 2048          # items per dense logit chunk inside a slice


def full_sum(name: str, threads: int) -> dict:
    p = W.draw_config(name, seed=SEED)
    bounds = [p.V * k // SLICES for k in range(SLICES + 1)]
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1, "blas")      # one BLAS thread per pool thread
    except ImportError:  # pragma: no cover
        limit = None
    t0 = time.time()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(lambda k: O.loss_sum_slice(p.H, p.E, p.targets, p.mask, bounds[k], bounds[k + 1],
                                                       chunk=CHUNK), range(SLICES)))
    if limit is not None:
        limit.unregister()
    total = 0.0
    for s in parts:                               # slice order: a fixed summation order
        total += s
    tg = O.positive_sets(p.targets, p.mask, p.V)
    return {"workload": name, "seed": SEED, "recipe": p.recipe, "T": p.T, "V": p.V, "D": p.D, "K": p.K,
            "n_valid": tg.n_valid, "n_pairs": tg.n_pairs, "sum_loss": total,
            "mean_loss": total / tg.n_valid, "slices": SLICES, "seconds": round(time.time() - t0, 1)}


def main(argv):
    names = argv or WORKLOADS
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = {e["workload"]: e for e in json.load(f)["entries"]}
    threads = os.cpu_count() or 1
    for name in names:
        e = full_sum(name, threads)
        print(json.dumps(e), flush=True)
        data[name] = e
        with open(OUT, "w") as f:
            json.dump({"what": "float64 oracle: sum over valid positions and all items of Eq. (2) "
                               "(reduction SUM), seed 0", "entries": [data[k] for k in WORKLOADS if k in data]},
                      f, indent=1)


if __name__ == "__main__":
    main(sys.argv[1:])
