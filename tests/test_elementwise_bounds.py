"""Host-side check of the reciprocals the tile engine uses for the sigmoid.

The kernels compute 1/w on the FMA pipe instead of the SFU: a seed, then one
cubically convergent step r1 = r0 (1 + e + e^2), e = 1 - w r0.
  * item pass, w in (1, 2]: linear minimax seed r0 = (24 - 8 w) / 17, one
    fused multiply-add on -w; bound (1/17)^3 = 2.1e-4;
  * gradient-only passes, w up to 2^100: exponent-flip seed
    r0 = bits^-1(C - bits(w)), C = 0x7EF31000 (formed from -w, whose bits are
    bits(w) + 2^31); bound 1.3e-4.
This test replays the same float32 operations (each fused multiply-add
rounded once, as on the GPU) over the ranges the kernels use.
"""
import numpy as np

SEED_NEG = np.uint32(0x7EF31000 + 0x80000000)


def fma32(a, b, c):
    # a*b of two float32 values is exact in float64; one rounding to float32 after the add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def rcp_cubic(w):
    w = np.asarray(w, np.float32)
    nw = -w
    r = (SEED_NEG - nw.view(np.uint32)).astype(np.uint32).view(np.float32)
    e = fma32(nw, r, np.float32(1.0))
    t = fma32(e, e, e)
    return fma32(r, t, r)


def rcp_linear_seed(w):
    w = np.asarray(w, np.float32)
    nw = -w
    r = fma32(nw, np.float32(8.0 / 17.0), np.float32(24.0 / 17.0))
    e = fma32(nw, r, np.float32(1.0))
    t = fma32(e, e, e)
    return fma32(r, t, r)


def test_reciprocal_bound_item_range():
    # item pass: w = 1 + e^{-|z|} in (1, 2]
    w = np.linspace(1.0, 2.0, 400001, dtype=np.float32)[1:]
    rel = np.abs(1.0 - w.astype(np.float64) * rcp_linear_seed(w).astype(np.float64))
    assert rel.max() <= (1.0 / 17.0) ** 3 + 1e-6, rel.max()
    # and the exponent-flip variant on the same range
    rel = np.abs(1.0 - w.astype(np.float64) * rcp_cubic(w).astype(np.float64))
    assert rel.max() <= 1.3e-4 + 1e-6, rel.max()


def test_reciprocal_bound_full_range():
    # gradient-only passes: w = 1 + 2^x with x clamped at 100
    x = np.linspace(-30.0, 100.0, 200001)
    w = (1.0 + np.exp2(x)).astype(np.float32)
    rel = np.abs(1.0 - w.astype(np.float64) * rcp_cubic(w).astype(np.float64))
    assert np.all(np.isfinite(rel))
    assert rel.max() <= 1.3e-4 + 1e-6, rel.max()


def test_seed_alone_is_within_five_percent():
    w = np.linspace(1.0, 2.0, 100001, dtype=np.float32)
    nw = -w
    r0 = (SEED_NEG - nw.view(np.uint32)).astype(np.uint32).view(np.float32)
    rel = np.abs(1.0 - w.astype(np.float64) * r0.astype(np.float64))
    assert rel.max() <= 0.0506, rel.max()
