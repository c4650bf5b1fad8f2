"""The C-ABI library without a GPU: it loads, exports every function
include/cutbce.h declares, and rejects bad arguments on the host before any
launch.  No compute call is made here."""
import ctypes
import subprocess

import pytest

from vocabulary_label_bce_b200 import binding as B


def _prob(T=12800, V=876000, D=64, K=16, dtype=B.BF16, red=0, ptrs=True):
    fake = 0x10000 if ptrs else None
    return B.cutbce_problem(T, V, D, K, dtype, red, fake, fake, fake, None)


def test_exports_every_declared_symbol():
    lib = B.load_library()
    declared = B.declared_functions()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", B.library_path()], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(declared) <= exported


def test_status_strings():
    assert B.cutbce_status_string(0) == "ok"
    assert "range" in B.cutbce_status_string(B.ERR_TARGET_RANGE)
    assert "wait" in B.cutbce_status_string(B.ERR_TIMEOUT)


def test_workspace_has_no_T_times_V_term():
    base = B.cutbce_workspace_size(_prob(V=100_000))
    big = B.cutbce_workspace_size(_prob(V=10_000_000))
    # growth in V is per item: one int offset into the item-sorted pairs, and per tile of
    # 128 items 16 double loss partials
    assert big - base <= (16 * 8 + 4 * 128) * (10_000_000 // 128 + 2) + 8192
    # and it is far below one [T, V] fp32 logit tensor
    assert big < 12800 * 10_000_000 * 4 / 100


@pytest.mark.parametrize("field,value,expect", [
    ("T", 0, B.ERR_INVALID_ARG), ("V", -1, B.ERR_INVALID_ARG), ("D", 60, B.ERR_UNSUPPORTED),
    ("D", 264, B.ERR_UNSUPPORTED), ("K", 129, B.ERR_UNSUPPORTED), ("dtype", 7, B.ERR_UNSUPPORTED),
    ("reduction", 5, B.ERR_INVALID_ARG),
])
def test_host_argument_errors(field, value, expect):
    p = _prob()
    setattr(p, field, value)
    with pytest.raises(B.CutBCEError) as e:
        B.cutbce_workspace_size(p)
    assert e.value.status == expect


def test_bf16_position_limit():
    # the item-owned pass packs a compacted position into 24 bits
    assert B.cutbce_workspace_size(_prob(T=(1 << 24) - 128, V=1000, K=1)) > 0
    with pytest.raises(B.CutBCEError) as e:
        B.cutbce_workspace_size(_prob(T=(1 << 24) - 127, V=1000, K=1))
    assert e.value.status == B.ERR_UNSUPPORTED
    # the fp32 path has no such limit
    assert B.cutbce_workspace_size(_prob(T=(1 << 24), V=1000, K=1, dtype=B.F32)) > 0


def test_compute_calls_reject_before_launch():
    lib = B.load_library()
    p = _prob(T=256, V=1000)
    n = ctypes.c_size_t()
    assert lib.cutbce_workspace_size_for(ctypes.byref(p), B.OUT_LOSS, ctypes.byref(n)) == 0
    loss = ctypes.c_void_p(0x20000)
    # null workspace, small workspace, misaligned workspace, null loss, null problem pointers
    assert lib.cutbce_forward(ctypes.byref(p), None, n.value, loss, None) == B.ERR_INVALID_ARG
    assert lib.cutbce_forward(ctypes.byref(p), ctypes.c_void_p(0x40000), n.value - 1, loss, None) == B.ERR_WORKSPACE
    assert lib.cutbce_forward(ctypes.byref(p), ctypes.c_void_p(0x40010), n.value, loss, None) == B.ERR_INVALID_ARG
    assert lib.cutbce_forward(ctypes.byref(p), ctypes.c_void_p(0x40000), n.value, None, None) == B.ERR_INVALID_ARG
    q = _prob(T=256, V=1000, ptrs=False)
    assert lib.cutbce_forward_backward(ctypes.byref(q), None, loss, None, None, ctypes.c_void_p(0x40000),
                                       n.value, None) == B.ERR_INVALID_ARG
    r = _prob(T=256, V=1000)
    r.H = 0x10002                                    # bf16 operands must be 16-byte aligned
    assert lib.cutbce_backward(ctypes.byref(r), None, ctypes.c_void_p(0x30000), None, ctypes.c_void_p(0x40000),
                               n.value, None) == B.ERR_INVALID_ARG
    assert lib.cutbce_backward(ctypes.byref(p), None, None, None, ctypes.c_void_p(0x40000), n.value,
                               None) == B.ERR_INVALID_ARG
    assert lib.cutbce_selftest_wait_timeout(0, ctypes.c_void_p(0x40000), None) == B.ERR_INVALID_ARG


def test_workspace_size_per_outputs():
    p = _prob()
    full = B.cutbce_workspace_size(p)
    assert full == B.cutbce_workspace_size_for(p, B.OUT_LOSS | B.OUT_DH | B.OUT_DE)
    loss_only = B.cutbce_workspace_size_for(p, B.OUT_LOSS)
    dh = B.cutbce_workspace_size_for(p, B.OUT_DH)
    de = B.cutbce_workspace_size_for(p, B.OUT_DE)
    assert loss_only < dh < full and loss_only < de < full
    # the loss-only layout holds neither the dH split partials nor the pair-sort buffers
    assert full - loss_only >= 16 * 12800 * 16 + 4 * 12800 * 64
    assert loss_only < 16 << 20
    met = B.cutbce_workspace_size_for(p, B.OUT_LOSS | B.OUT_METRICS)
    assert met - loss_only >= 8 * 12800            # one (count, TP) pair per position and split slot
    for bad in (0, 16, -1):
        with pytest.raises(B.CutBCEError) as e:
            B.cutbce_workspace_size_for(p, bad)
        assert e.value.status == B.ERR_INVALID_ARG


def test_launch_accounting():
    p = _prob()
    # rows, scan, gather, column sums of E and of H_c, sort keys, 2 radix passes x 3
    # (6844 item tiles: 13-bit keys), item-tile offsets, item pass, dH pass, finish
    assert B.cutbce_kernel_launches(p, 2) == 16
    assert B.cutbce_kernel_launches(p, 0) == 7          # rows, scan, gather, 2 column sums, item pass, finish
    assert B.cutbce_kernel_launches(p, 1) == 14         # backward: no loss, so no column sums
    assert B.cutbce_kernel_launches(p, 3) == -1


def test_host_buffer_size_covers_inputs_and_outputs():
    p = _prob(T=1000, V=5000)
    need = B.cutbce_host_buffer_size(p)
    ws = B.cutbce_workspace_size(p)
    assert need >= ws + 1000 * 64 * (2 + 4) + 5000 * 64 * (2 + 4) + 1000 * 16 * 4
