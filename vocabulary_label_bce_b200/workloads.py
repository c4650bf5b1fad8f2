"""Seeded synthetic inputs for the fused large-vocabulary BCE loss.

This module only draws random inputs. It holds none of the loss arithmetic,
so both the CUDA path and the float64 oracle may take their inputs from it.

The shapes and distributions follow the workloads of "Cut Binary Cross
Entropy: Efficient Large-Vocabulary Loss and Gradient Kernels for Sequential
Recommendation" (section IV-A mini-benchmark: A ~ N(0, I), E ~ N(0, I),
uniform target ids; section IV-B: multi-label SASRec on Yambda-50M with
V = 876,939 items).  No dataset is used: every input is drawn here, from
numpy's PCG64 with one SeedSequence child stream per input, so that the same
seed always gives the same bits.

Layout of a drawn problem (all numpy, host memory):
  H        float32 [T, D]   values exactly representable in bf16 (or plain
                            fp32 for dtype "f32")
  H_bits   uint16  [T, D]   the bf16 bit patterns of H (None for "f32")
  E, E_bits                 the same for the item table [V, D]
  targets  int32   [T, K]   positive item ids, -1 marks an empty slot
  mask     uint8   [T]      1 = valid position, 0 = padding
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = ["Problem", "CONFIGS", "draw", "draw_config", "to_bf16_bits", "bf16_bits_to_f32"]

_E_CHUNK_ROWS = 1 << 16


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); return the bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to the float32 values they stand for (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Problem:
    name: str
    B: int
    N: int
    T: int
    V: int
    D: int
    K: int
    dtype: str                  # "bf16" or "f32"
    H: np.ndarray
    E: np.ndarray
    targets: np.ndarray
    mask: np.ndarray
    H_bits: Optional[np.ndarray] = None
    E_bits: Optional[np.ndarray] = None
    recipe: str = ""

    @property
    def n_valid(self) -> int:
        return int(self.mask.astype(bool).sum())


def _zipf_cdf(V: int, s: float) -> np.ndarray:
    # bounded Zipf over ranks r = 0..V-1 with p(r) proportional to (r+1)^-s; item id = rank
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def _distinct_ids(rng: np.random.Generator, counts: np.ndarray, V: int, zipf_s: Optional[float],
                  K: int) -> np.ndarray:
    """Draw counts[t] distinct ids per row (rejection of repeats), pad with -1 to K slots."""
    T = counts.shape[0]
    out = np.full((T, K), -1, dtype=np.int32)
    cdf = _zipf_cdf(V, zipf_s) if zipf_s is not None else None

    def sample(n):
        if cdf is None:
            return rng.integers(0, V, size=n, dtype=np.int64)
        u = rng.random(n)
        return np.minimum(np.searchsorted(cdf, u, side="right"), V - 1)

    for t in range(T):
        need = int(counts[t])
        if need == 0:
            continue
        if need > V:
            raise ValueError("more distinct ids requested than items")
        got: list[int] = []
        seen: set[int] = set()
        while len(got) < need:
            for x in sample(2 * (need - len(got)) + 2).tolist():
                if x not in seen:
                    seen.add(x)
                    got.append(x)
                    if len(got) == need:
                        break
        out[t, :need] = np.asarray(got, dtype=np.int32)
    return out


def _draw_normal_rows(rng: np.random.Generator, rows: int, D: int, std: float) -> np.ndarray:
    out = np.empty((rows, D), dtype=np.float32)
    for r0 in range(0, rows, _E_CHUNK_ROWS):
        r1 = min(rows, r0 + _E_CHUNK_ROWS)
        out[r0:r1] = rng.standard_normal((r1 - r0, D), dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def draw(*, T: int, V: int, D: int, K: int, B: Optional[int] = None, N: Optional[int] = None,
         dtype: str = "bf16", seed: int = 0, h_std: float = 1.0, e_std: Optional[float] = None,
         count: str = "full", count_mean: float = 3.0, count_max: Optional[int] = None,
         ids: str = "uniform", zipf_s: float = 1.1,
         mask: str = "random", mask_frac: float = 0.0, trailing: int = 0,
         name: str = "custom") -> Problem:
    """Draw one problem.

    count: "full" (K ids per row), "poisson" (Poisson(count_mean) clipped to [1, count_max]).
    ids:   "uniform" over [0, V) or "zipf" (bounded Zipf with exponent zipf_s, id = rank).
    mask:  "random" (exactly round(mask_frac*T) rows masked, uniform without replacement),
           "trailing" (the last `trailing` positions of every length-N sequence masked),
           "none".
    E rows are N(0, e_std^2), e_std defaulting to 1/sqrt(D); H rows are N(0, h_std^2).
    """
    if B is None or N is None:
        B, N = 1, T
    assert B * N == T
    if e_std is None:
        e_std = 1.0 / np.sqrt(D)
    ss = np.random.SeedSequence(seed)
    r_h, r_e, r_cnt, r_ids, r_mask = [np.random.Generator(np.random.PCG64(c)) for c in ss.spawn(5)]

    H = _draw_normal_rows(r_h, T, D, h_std)
    E = _draw_normal_rows(r_e, V, D, e_std)

    if count == "full":
        counts = np.full(T, K, dtype=np.int64)
    elif count == "poisson":
        cmax = K if count_max is None else count_max
        counts = np.clip(r_cnt.poisson(count_mean, size=T), 1, cmax)
    else:
        raise ValueError(count)
    targets = _distinct_ids(r_ids, counts, V, zipf_s if ids == "zipf" else None, K)

    m = np.ones(T, dtype=np.uint8)
    if mask == "random":
        n_masked = int(round(mask_frac * T))
        if n_masked:
            m[r_mask.choice(T, size=n_masked, replace=False)] = 0
    elif mask == "trailing":
        m.reshape(B, N)[:, N - trailing:] = 0
    elif mask != "none":
        raise ValueError(mask)

    H_bits = E_bits = None
    if dtype == "bf16":
        H_bits = to_bf16_bits(H)
        E_bits = to_bf16_bits(E)
        H = bf16_bits_to_f32(H_bits)
        E = bf16_bits_to_f32(E_bits)
    elif dtype != "f32":
        raise ValueError(dtype)
    recipe = (f"seed={seed} T={T} (B={B},N={N}) V={V} D={D} K={K} {dtype}; H~N(0,{h_std}^2), "
              f"E~N(0,{e_std:.4g}^2); counts={count}; ids={ids}"
              + (f"(s={zipf_s})" if ids == "zipf" else "") + f"; mask={mask}")
    return Problem(name=name, B=B, N=N, T=T, V=V, D=D, K=K, dtype=dtype, H=H, E=E,
                   targets=targets, mask=m, H_bits=H_bits, E_bits=E_bits, recipe=recipe)


# The five workloads, by what they are and their sizes.
CONFIGS = {
    "tiny_f32": dict(T=64, B=4, N=16, D=32, V=2048, K=4, dtype="f32", count="full",
                     ids="uniform", mask="random", mask_frac=0.10),
    "small_catalog": dict(T=6400, B=32, N=200, D=64, V=100_000, K=8, dtype="bf16",
                          count="full", ids="zipf", zipf_s=1.1, mask="trailing", trailing=30),
    "sasrec_876k": dict(T=12800, B=64, N=200, D=64, V=876_000, K=16, dtype="bf16",
                        count="poisson", count_mean=3.0, count_max=16, ids="zipf", zipf_s=1.05,
                        mask="trailing", trailing=40),
    "wide_d256": dict(T=8192, B=16, N=512, D=256, V=1_000_000, K=16, dtype="bf16",
                      count="full", ids="zipf", zipf_s=1.1, mask="random", mask_frac=0.10),
    "extreme_10m": dict(T=4096, B=8, N=512, D=128, V=10_000_000, K=4, dtype="bf16",
                        count="full", ids="uniform", mask="random", mask_frac=0.05),
}


def draw_config(name: str, seed: int = 0) -> Problem:
    return draw(name=name, seed=seed, **CONFIGS[name])
