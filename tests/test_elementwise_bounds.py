"""Host-side replay of the FMA-pipe element math of the tile engine.

The gradient-only passes evaluate two pairs of logits in 16 wholly on the FMA
pipe: 2^x by a degree-3 polynomial with integer exponent insertion, then 1/w
by the exponent-flip seed r0 = bits^-1(C - bits(w)), C = 0x7EF31000 (formed
from -w, whose bits are bits(w) + 2^31), and one cubically convergent step
r1 = r0 (1 + e + e^2), e = 1 - w r0, which leaves |e|^3 <= 1.3e-4.
These tests replay the same float32 operations (each fused multiply-add
rounded once, as on the GPU) over the ranges the kernels use; the GPU test of
the element-math self test checks the device against this replay bit for bit.
The SFU paths (ex2, tanh) are checked on the device against their bounds.
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


def test_reciprocal_bound_unit_range():
    # w in (1, 2]
    w = np.linspace(1.0, 2.0, 400001, dtype=np.float32)[1:]
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


# ---------------------------------------------------------------- FMA-pipe sigmoid of the gradient-only passes
# The same float32 operations as exp2_poly3_pair and sigmoid_pair_fma (each fused
# multiply-add rounded once; the integer exponent insertion as a 32-bit
# multiply-add), replayed over the clamped input range.
POLY3 = [np.float32(v) for v in (0.9999280572, 0.6932609677, 0.2426111251, 0.0551716685)]
SHIFT = np.float32(12582912.0)            # 1.5 * 2^23
LOG2E = np.float32(1.4426950408889634)


def add32(a, b):
    return (np.asarray(a, np.float32).astype(np.float64) + np.asarray(b, np.float32).astype(np.float64)).astype(np.float32)


def exp2_poly3(x):
    x = np.asarray(x, np.float32)
    j = add32(x, SHIFT)
    jr = add32(j, -SHIFT)
    f = fma32(jr, np.float32(-1.0), x)
    p = fma32(np.full_like(f, POLY3[3]), f, np.full_like(f, POLY3[2]))
    p = fma32(p, f, np.full_like(f, POLY3[1]))
    p = fma32(p, f, np.full_like(f, POLY3[0]))
    bits = (j.view(np.uint32).astype(np.uint64) * (1 << 23) + p.view(np.uint32).astype(np.uint64)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def sat(v):
    return np.clip(v, np.float32(0.0), np.float32(1.0)).astype(np.float32)


def sigmoid_fma(z):
    z = np.asarray(z, np.float32)
    a = sat(fma32(z, np.float32(-LOG2E / np.float32(200.0)), np.float32(0.5)))
    x = fma32(a, np.float32(200.0), np.float32(-100.0))
    v = exp2_poly3(x)
    nw = fma32(v, np.float32(-1.0), np.float32(-1.0))
    return rcp_cubic(-nw)


def test_exp2_poly3_bound():
    x = np.linspace(-100.0, 100.0, 2000001).astype(np.float32)
    got = exp2_poly3(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert np.all(np.isfinite(got))
    assert rel.max() <= 7.6e-5, rel.max()
    # the polynomial's own fit, without the range reduction, at its extremes
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    assert np.abs(exp2_poly3(f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max() <= 7.6e-5


def test_gradient_only_sigmoid_bound():
    z = np.concatenate([np.linspace(-69.0, 69.0, 400001), np.linspace(-8.0, 8.0, 200001)]).astype(np.float32)
    ref = 1.0 / (1.0 + np.exp(-z.astype(np.float64)))
    got = sigmoid_fma(z).astype(np.float64)
    rel = np.abs(got / ref - 1.0)
    # clamp 4e-6 relative in 2^x (at most that in sigmoid) + polynomial 7.5e-5 + reciprocal 1.3e-4
    assert rel.max() <= 2.1e-4, rel.max()
    # beyond the clamp the result stays positive and tiny instead of underflowing to garbage
    far = sigmoid_fma(np.array([-80.0, -500.0, -3e38], np.float32))
    assert np.all(far > 0) and np.all(far < 1e-29)
    assert np.all(sigmoid_fma(np.array([80.0, 3e38], np.float32)) > np.float32(0.9998))
