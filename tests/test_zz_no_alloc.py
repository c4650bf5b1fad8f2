"""The fixed-scratch forward entry (cutbce_forward_fixed_scratch) through the
C ABI: it allocates nothing, takes no workspace, and must give the loss of
cutbce_forward on the same problem.  Named so that it is collected last: it
has to pass both alone and after every other test has used the library."""
import ctypes
import math

import numpy as np
import pytest
import torch

from vocabulary_label_bce_b200 import binding as B
from vocabulary_label_bce_b200 import workloads as W

from gpu_util import to_device


def _fits(prob):
    return B.cutbce_workspace_size_for(prob, B.OUT_LOSS) <= B.FIXED_SCRATCH_BYTES


def test_header_constant_matches_binding():
    import re
    text = open(B._HEADER).read()
    m = re.search(r"#define CUTBCE_FIXED_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == B.FIXED_SCRATCH_BYTES


def test_rejects_problems_beyond_the_fixed_scratch():
    # host-side rejection, before any device call: fake device pointers are never touched
    lib = B.load_library()
    fake = 0x10000
    prob = B.cutbce_problem(200_000, 1000, 64, 16, B.BF16, 0, fake, fake, fake, None)
    assert not _fits(prob)
    st = lib.cutbce_forward_fixed_scratch(ctypes.byref(prob), fake, None)
    assert st == B.ERR_WORKSPACE
    assert lib.cutbce_forward_fixed_scratch(ctypes.byref(prob), None, None) == B.ERR_INVALID_ARG


def test_workload_sizes_fit():
    # the loss-only workspace of the small catalog and of the SASRec-style head fit the array
    fake = 0x10000
    for name in ("small_catalog", "sasrec_876k"):
        c = W.CONFIGS[name]
        prob = B.cutbce_problem(c["T"], c["V"], c["D"], c["K"], B.BF16, 0, fake, fake, fake, None)
        assert _fits(prob), name


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [dict(T=333, V=1500, D=64, K=4), dict(T=200, V=777, D=256, K=16),
                                   dict(T=129, V=640, D=96, K=3), "small_catalog"],
                         ids=lambda s: s if isinstance(s, str) else f"T{s['T']}_V{s['V']}_D{s['D']}")
def test_fixed_scratch_matches_workspace_entry(shape):
    if isinstance(shape, str):
        p = W.draw_config(shape, seed=0)
    else:
        p = W.draw(**shape, dtype="bf16", seed=11, ids="zipf", zipf_s=1.1, mask="random", mask_frac=0.1)
    H, E, tg, m = to_device(p)
    prob = B.make_problem(H, E, tg, m, "mean")
    assert _fits(prob)
    # the existing entry, with a caller workspace
    ws = torch.empty(B.cutbce_workspace_size_for(prob, B.OUT_LOSS), dtype=torch.uint8, device="cuda")
    ref = torch.full((), float("nan"), dtype=torch.float64, device="cuda")
    B.cutbce_forward(prob, ws, ref)
    assert B.cutbce_read_status(ws) == 0
    ref_loss = float(ref.item())
    assert math.isfinite(ref_loss)
    # the fixed-scratch entry, twice in a row on the same stream: the same kernels
    # run in the same order on the same workspace layout, so the loss is identical
    for _ in range(2):
        got = torch.full((), float("nan"), dtype=torch.float64, device="cuda")
        B.cutbce_forward_fixed_scratch(prob, got)
        torch.cuda.synchronize()
        g = float(got.item())
        assert g == ref_loss, (g, ref_loss)
