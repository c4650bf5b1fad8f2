"""ctypes binding of libcutbce (include/cutbce.h): argument marshalling only.

Every step of the loss and its gradient runs in the library's CUDA kernels;
this module only turns torch tensors into pointers and sizes, takes the
current CUDA stream, and allocates outputs and the workspace through torch.
There is no CPU fallback: if the library is missing, importing a function that
needs it raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

__all__ = [
    "CutBCEError", "cutbce_problem", "load_library", "library_path", "declared_functions",
    "cutbce_workspace_size", "cutbce_workspace_size_for", "OUT_LOSS", "OUT_DH", "OUT_DE", "OUT_METRICS",
    "cutbce_options", "make_options", "cutbce_forward_backward_ex", "cutbce_workspace_size_ex",
    "GRAD_F32", "GRAD_BF16", "ACCUMULATE_DH", "ACCUMULATE_DE", "cutbce_forward", "cutbce_forward_fixed_scratch", "FIXED_SCRATCH_BYTES",
    "cutbce_backward", "cutbce_forward_backward",
    "cutbce_host_buffer_size", "cutbce_forward_backward_host", "cutbce_read_status",
    "cutbce_read_counts", "cutbce_kernel_launches", "cutbce_status_string",
    "cutbce_selftest_wait_timeout", "cutbce_selftest_element_math", "cutbce_topk_workspace_size", "cutbce_topk",
    "cutbce_hit_at_k", "cutbce_profile_enable", "cutbce_profile_read", "REDUCTIONS",
    "KERNEL_KINDS", "cutbce_probe_scratch_bytes", "cutbce_probe_pipe_rate", "PROBES", "cutbce_probe_mma",
]

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_TARGET_RANGE, ERR_TIMEOUT, ERR_CUDA = range(7)
BF16, F32 = 0, 1
OUT_LOSS, OUT_DH, OUT_DE, OUT_METRICS = 1, 2, 4, 8
REDUCTIONS = {"mean": 0, "sum": 1, "mean_elements": 2}

_PKG = os.path.dirname(os.path.abspath(__file__))
_HEADER = os.path.join(os.path.dirname(_PKG), "include", "cutbce.h")


def library_path() -> str:
    return os.path.join(_PKG, "libcutbce.so")


class cutbce_problem(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64), ("V", ctypes.c_int64), ("D", ctypes.c_int64), ("K", ctypes.c_int64),
        ("dtype", ctypes.c_int32), ("reduction", ctypes.c_int32),
        ("H", ctypes.c_void_p), ("E", ctypes.c_void_p), ("targets", ctypes.c_void_p), ("mask", ctypes.c_void_p),
    ]


class cutbce_options(ctypes.Structure):
    _fields_ = [("metrics", ctypes.c_void_p), ("weights", ctypes.c_void_p), ("grad_dtype", ctypes.c_int32),
                ("accumulate", ctypes.c_int32), ("vocab_offset", ctypes.c_int64), ("V_total", ctypes.c_int64)]


GRAD_F32, GRAD_BF16 = 0, 1
ACCUMULATE_DH, ACCUMULATE_DE = 1, 2


def make_options(metrics: Optional[torch.Tensor] = None, weights: Optional[torch.Tensor] = None,
                 grad_dtype: int = GRAD_F32, accumulate: int = 0, vocab_offset: int = 0,
                 V_total: int = 0) -> cutbce_options:
    """Options of cutbce_forward_backward_ex (see include/cutbce.h): metrics is an int32 [T, 4]
    device tensor, weights a float32 [T] device tensor."""
    if metrics is not None and (metrics.dtype != torch.int32 or not metrics.is_contiguous()):
        raise ValueError("metrics must be a contiguous int32 [T, 4] tensor")
    if weights is not None and (weights.dtype != torch.float32 or not weights.is_contiguous()):
        raise ValueError("weights must be a contiguous float32 [T] tensor")
    return cutbce_options(metrics.data_ptr() if metrics is not None else None,
                          weights.data_ptr() if weights is not None else None,
                          int(grad_dtype), int(accumulate), int(vocab_offset), int(V_total))


class CutBCEError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        msg = _LIB.cutbce_status_string(self.status).decode() if _LIB is not None else str(status)
        super().__init__(f"{where}: {msg} (status {self.status})" if where else f"{msg} (status {self.status})")


_LIB: Optional[ctypes.CDLL] = None
_P = ctypes.POINTER(cutbce_problem)
_vp, _sz, _i32, _i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
_SIGS = {
    "cutbce_workspace_size": (_i32, [_P, ctypes.POINTER(_sz)]),
    "cutbce_workspace_size_for": (_i32, [_P, ctypes.c_int, ctypes.POINTER(_sz)]),
    "cutbce_forward": (_i32, [_P, _vp, _sz, _vp, _vp]),
    "cutbce_forward_fixed_scratch": (_i32, [_P, _vp, _vp]),
    "cutbce_backward": (_i32, [_P, _vp, _vp, _vp, _vp, _sz, _vp]),
    "cutbce_forward_backward": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "cutbce_forward_backward_ex": (_i32, [_P, ctypes.POINTER(cutbce_options), _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "cutbce_workspace_size_ex": (_i32, [_P, ctypes.POINTER(cutbce_options), ctypes.c_int, ctypes.POINTER(_sz)]),
    "cutbce_host_buffer_size": (_i32, [_P, ctypes.POINTER(_sz)]),
    "cutbce_forward_backward_host": (_i32, [_P, ctypes.c_float, _vp, _vp, _vp, _vp, _sz, _vp]),
    "cutbce_read_status": (_i32, [_vp, _vp]),
    "cutbce_read_counts": (_i32, [_P, _vp, ctypes.POINTER(_i64), ctypes.POINTER(_i64), _vp, _vp]),
    "cutbce_kernel_launches": (ctypes.c_int, [_P, ctypes.c_int]),
    "cutbce_status_string": (ctypes.c_char_p, [_i32]),
    "cutbce_selftest_wait_timeout": (_i32, [_i64, _vp, _vp]),
    "cutbce_selftest_element_math": (_i32, [_vp, _vp, _i64, _vp]),
    "cutbce_topk_workspace_size": (_i32, [_i64, _i64, _i64, ctypes.c_int, ctypes.POINTER(_sz)]),
    "cutbce_topk": (_i32, [_vp, _i64, _vp, _i64, _i64, _i32, ctypes.c_int, _vp, _vp, _vp, _sz, _vp]),
    "cutbce_hit_at_k": (_i32, [_vp, _i64, ctypes.c_int, _vp, _i64, _vp, _vp]),
    "cutbce_profile_enable": (_i32, [ctypes.c_int]),
    "cutbce_profile_read": (_i32, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64), ctypes.c_int]),
    "cutbce_probe_scratch_bytes": (_sz, []),
    "cutbce_probe_pipe_rate": (_i32, [ctypes.c_int, _vp, _sz, ctypes.POINTER(ctypes.c_double), _vp]),
    "cutbce_probe_mma": (_i32, [ctypes.c_int, ctypes.c_int, _i64, _vp, _sz, ctypes.POINTER(ctypes.c_double),
                                ctypes.POINTER(ctypes.c_double), _vp]),
}
PROBES = ["ffma", "ffma2", "ex2", "rcp", "tanh", "lg2", "cvt_bf16x2", "fmax", "add2", "iadd", "prmt",
          "ex2_f16x2", "ex2_bf16x2", "tanh_f16x2", "hfma2", "cvt_f16x2", "ffma_sat", "select", "lop", "fmul2"]
KERNEL_KINDS = ["prep_rows", "prep_scan", "prep_gather", "csc_offsets", "item_pass", "position_pass", "finish",
                "pair_sort", "topk", "topk_merge", "col_sums"]


def load_library() -> ctypes.CDLL:
    """Load the in-tree libcutbce.so (built by `python -m vocabulary_label_bce_b200.build`)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m vocabulary_label_bce_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def declared_functions() -> list[str]:
    """Names of the functions include/cutbce.h declares."""
    text = open(_HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cutbce_[a-z_]+)\s*\(", text)))


def _check(status: int, where: str) -> None:
    if status != OK:
        raise CutBCEError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_problem(H: torch.Tensor, E: torch.Tensor, targets: torch.Tensor, mask: Optional[torch.Tensor] = None,
                 reduction: str | int = "mean") -> cutbce_problem:
    """Describe tensors already on the device.  H [T, D], E [V, D] bf16 or fp32, targets int32 [T, K]."""
    if H.dim() != 2 or E.dim() != 2 or targets.dim() != 2:
        raise ValueError("H, E, targets must be 2-D")
    if H.dtype != E.dtype or H.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("H and E must share dtype bf16 or fp32")
    if targets.dtype != torch.int32:
        raise ValueError("targets must be int32")
    for t in (H, E, targets) + ((mask,) if mask is not None else ()):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    if mask is not None and mask.dtype not in (torch.uint8, torch.bool):
        raise ValueError("mask must be uint8 or bool")
    red = REDUCTIONS[reduction] if isinstance(reduction, str) else int(reduction)
    return cutbce_problem(H.shape[0], E.shape[0], H.shape[1], targets.shape[1],
                          BF16 if H.dtype == torch.bfloat16 else F32, red,
                          H.data_ptr(), E.data_ptr(), targets.data_ptr(),
                          mask.data_ptr() if mask is not None else None)


# ---------------------------------------------------------------- one function per C entry point
def cutbce_workspace_size(prob: cutbce_problem) -> int:
    n = _sz(0)
    _check(load_library().cutbce_workspace_size(ctypes.byref(prob), ctypes.byref(n)), "cutbce_workspace_size")
    return int(n.value)


def cutbce_workspace_size_for(prob: cutbce_problem, outputs: int) -> int:
    """Workspace bytes for a call computing only `outputs` (a bitwise or of OUT_LOSS, OUT_DH, OUT_DE)."""
    n = _sz(0)
    _check(load_library().cutbce_workspace_size_for(ctypes.byref(prob), int(outputs), ctypes.byref(n)),
           "cutbce_workspace_size_for")
    return int(n.value)


def cutbce_workspace_size_ex(prob: cutbce_problem, opts: Optional[cutbce_options], outputs: int) -> int:
    n = _sz(0)
    _check(load_library().cutbce_workspace_size_ex(ctypes.byref(prob), ctypes.byref(opts) if opts is not None else None,
                                                   int(outputs), ctypes.byref(n)), "cutbce_workspace_size_ex")
    return int(n.value)


def cutbce_forward(prob, ws: torch.Tensor, loss: torch.Tensor, stream=None) -> None:
    _check(load_library().cutbce_forward(ctypes.byref(prob), ws.data_ptr(), ws.numel(), loss.data_ptr(),
                                         _stream(stream)), "cutbce_forward")


# Size of the library's static scratch array (CUTBCE_FIXED_SCRATCH_BYTES in include/cutbce.h).
FIXED_SCRATCH_BYTES = 16 << 20


def cutbce_forward_fixed_scratch(prob, loss: torch.Tensor, stream=None) -> None:
    """Loss only, with the library's static scratch array instead of a workspace (nothing is allocated)."""
    _check(load_library().cutbce_forward_fixed_scratch(ctypes.byref(prob), loss.data_ptr(), _stream(stream)),
           "cutbce_forward_fixed_scratch")


def cutbce_backward(prob, grad_loss: Optional[torch.Tensor], dH: Optional[torch.Tensor],
                    dE: Optional[torch.Tensor], ws: torch.Tensor, stream=None) -> None:
    _check(load_library().cutbce_backward(
        ctypes.byref(prob), grad_loss.data_ptr() if grad_loss is not None else None,
        dH.data_ptr() if dH is not None else None, dE.data_ptr() if dE is not None else None,
        ws.data_ptr(), ws.numel(), _stream(stream)), "cutbce_backward")


def cutbce_forward_backward(prob, grad_loss: Optional[torch.Tensor], loss: Optional[torch.Tensor],
                            dH: Optional[torch.Tensor], dE: Optional[torch.Tensor], ws: torch.Tensor,
                            stream=None) -> None:
    _check(load_library().cutbce_forward_backward(
        ctypes.byref(prob), grad_loss.data_ptr() if grad_loss is not None else None,
        loss.data_ptr() if loss is not None else None, dH.data_ptr() if dH is not None else None,
        dE.data_ptr() if dE is not None else None, ws.data_ptr(), ws.numel(), _stream(stream)),
        "cutbce_forward_backward")


def cutbce_forward_backward_ex(prob, opts: cutbce_options, grad_loss: Optional[torch.Tensor],
                               loss: Optional[torch.Tensor], dH: Optional[torch.Tensor], dE: Optional[torch.Tensor],
                               ws: torch.Tensor, stream=None) -> None:
    _check(load_library().cutbce_forward_backward_ex(
        ctypes.byref(prob), ctypes.byref(opts), grad_loss.data_ptr() if grad_loss is not None else None,
        loss.data_ptr() if loss is not None else None, dH.data_ptr() if dH is not None else None,
        dE.data_ptr() if dE is not None else None, ws.data_ptr(), ws.numel(), _stream(stream)),
        "cutbce_forward_backward_ex")


def cutbce_host_buffer_size(prob: cutbce_problem) -> int:
    n = _sz(0)
    _check(load_library().cutbce_host_buffer_size(ctypes.byref(prob), ctypes.byref(n)), "cutbce_host_buffer_size")
    return int(n.value)


def cutbce_forward_backward_host(prob, grad_loss: float, loss: torch.Tensor, dH: Optional[torch.Tensor],
                                 dE: Optional[torch.Tensor], dev_buf: torch.Tensor, stream=None) -> None:
    """prob's pointers and loss/dH/dE are host (CPU, ideally pinned) tensors; dev_buf is device memory."""
    _check(load_library().cutbce_forward_backward_host(
        ctypes.byref(prob), float(grad_loss), loss.data_ptr(), dH.data_ptr() if dH is not None else None,
        dE.data_ptr() if dE is not None else None, dev_buf.data_ptr(), dev_buf.numel(), _stream(stream)),
        "cutbce_forward_backward_host")


def cutbce_read_status(ws: torch.Tensor, stream=None) -> int:
    return int(load_library().cutbce_read_status(ws.data_ptr(), _stream(stream)))


def cutbce_read_counts(prob, ws: torch.Tensor, row_counts: Optional[torch.Tensor] = None, stream=None):
    nv, npairs = _i64(0), _i64(0)
    _check(load_library().cutbce_read_counts(ctypes.byref(prob), ws.data_ptr(), ctypes.byref(nv),
                                             ctypes.byref(npairs),
                                             row_counts.data_ptr() if row_counts is not None else None,
                                             _stream(stream)), "cutbce_read_counts")
    return int(nv.value), int(npairs.value)


def cutbce_kernel_launches(prob, entry: int) -> int:
    return int(load_library().cutbce_kernel_launches(ctypes.byref(prob), int(entry)))


def cutbce_status_string(status: int) -> str:
    return load_library().cutbce_status_string(int(status)).decode()


def cutbce_selftest_wait_timeout(limit_ns: int, status_dev: torch.Tensor, stream=None) -> None:
    _check(load_library().cutbce_selftest_wait_timeout(int(limit_ns), status_dev.data_ptr(), _stream(stream)),
           "cutbce_selftest_wait_timeout")


def cutbce_selftest_element_math(x: torch.Tensor, stream=None) -> torch.Tensor:
    """[5, n] device tensor: FMA-pipe 2^x, SFU 2^x, FMA-pipe sigmoid(x), sigmoid(x) from
    tanh, and w = 1 + |tanh(x/2)| (see include/cutbce.h)."""
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 tensor")
    out = torch.empty((5, x.numel()), dtype=torch.float32, device=x.device)
    _check(load_library().cutbce_selftest_element_math(x.data_ptr(), out.data_ptr(), x.numel(), _stream(stream)),
           "cutbce_selftest_element_math")
    return out


def cutbce_topk_workspace_size(B: int, V: int, D: int, k: int) -> int:
    n = _sz(0)
    _check(load_library().cutbce_topk_workspace_size(int(B), int(V), int(D), int(k), ctypes.byref(n)),
           "cutbce_topk_workspace_size")
    return int(n.value)


def cutbce_topk(Q: torch.Tensor, E: torch.Tensor, k: int, ws: Optional[torch.Tensor] = None, stream=None):
    """(ids int32 [B, k], scores float32 [B, k]) of the k best items of every query row of Q (bf16 [B, D])."""
    if Q.dtype != torch.bfloat16 or E.dtype != torch.bfloat16 or not (Q.is_contiguous() and E.is_contiguous()):
        raise ValueError("Q and E must be contiguous bf16 tensors")
    B, D = Q.shape
    V = E.shape[0]
    if ws is None:
        ws = torch.empty(cutbce_topk_workspace_size(B, V, D, k), dtype=torch.uint8, device=Q.device)
    ids = torch.empty((B, k), dtype=torch.int32, device=Q.device)
    scores = torch.empty((B, k), dtype=torch.float32, device=Q.device)
    _check(load_library().cutbce_topk(Q.data_ptr(), B, E.data_ptr(), V, D, BF16, int(k), ids.data_ptr(),
                                      scores.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)), "cutbce_topk")
    return ids, scores


def cutbce_hit_at_k(ids: torch.Tensor, targets: torch.Tensor, stream=None) -> torch.Tensor:
    """int32 [B]: 1 where one of the query's target ids (-1 = empty) is among its ranked ids."""
    B, k = ids.shape
    hits = torch.empty(B, dtype=torch.int32, device=ids.device)
    _check(load_library().cutbce_hit_at_k(ids.data_ptr(), B, int(k), targets.data_ptr(), targets.shape[1],
                                          hits.data_ptr(), _stream(stream)), "cutbce_hit_at_k")
    return hits


def cutbce_profile_enable(enable: bool) -> None:
    _check(load_library().cutbce_profile_enable(1 if enable else 0), "cutbce_profile_enable")


def cutbce_profile_read(reset: bool = True) -> dict:
    """{kernel kind: (total ms, launches)} accumulated since the last reset."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (_i64 * n)()
    _check(load_library().cutbce_profile_read(ms, cnt, 1 if reset else 0), "cutbce_profile_read")
    return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}


def cutbce_probe_scratch_bytes() -> int:
    return int(load_library().cutbce_probe_scratch_bytes())


def cutbce_probe_pipe_rate(op: str | int, scratch: Optional[torch.Tensor] = None, stream=None) -> float:
    """Operations of one kind an SM retires per clock (median over SMs)."""
    k = PROBES.index(op) if isinstance(op, str) else int(op)
    if scratch is None:
        scratch = torch.empty(cutbce_probe_scratch_bytes(), dtype=torch.uint8, device="cuda")
    r = ctypes.c_double(0.0)
    _check(load_library().cutbce_probe_pipe_rate(k, scratch.data_ptr(), scratch.numel(), ctypes.byref(r),
                                                 _stream(stream)), "cutbce_probe_pipe_rate")
    return float(r.value)


def cutbce_probe_mma(n: int, a_in_tmem: bool, iters: int = 4096, scratch: Optional[torch.Tensor] = None,
                     stream=None, b_mn_major: bool = False, sm_pair: bool = False) -> tuple[float, float]:
    """(issue cycles, total cycles) per 128 x n x 16 bf16 tcgen05.mma (256 x n x 16
    over an SM pair if sm_pair), median over the issuing CTAs."""
    if scratch is None:
        scratch = torch.empty(cutbce_probe_scratch_bytes(), dtype=torch.uint8, device="cuda")
    a, b = ctypes.c_double(0.0), ctypes.c_double(0.0)
    flags = (1 if a_in_tmem else 0) | (2 if b_mn_major else 0) | (4 if sm_pair else 0)
    _check(load_library().cutbce_probe_mma(int(n), flags, int(iters), scratch.data_ptr(),
                                           scratch.numel(), ctypes.byref(a), ctypes.byref(b), _stream(stream)),
           "cutbce_probe_mma")
    return float(a.value), float(b.value)
