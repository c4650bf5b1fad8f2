"""B200-native exact fused large-vocabulary binary cross-entropy (loss and gradient).

C ABI: include/cutbce.h (libcutbce.so, built in-tree for sm_100a).
Python: `binding` mirrors the C entry points one to one; `api` offers
torch-facing calls and an autograd-aware `cut_bce`.
"""
from . import workloads  # noqa: F401  (seeded synthetic inputs; no loss arithmetic)

__all__ = ["workloads", "binding", "api"]


def __getattr__(name):
    # the binding and api need torch and the built library; import them lazily
    if name in ("binding", "api"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
