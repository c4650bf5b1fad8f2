"""The seeded input generator: determinism, shapes and the stated distributions."""
import numpy as np
import pytest

from vocabulary_label_bce_b200 import workloads as W


def test_bf16_rounding_rne():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 2**-7, 1.0 + 3 * 2**-8, -2.5, 0.0, 3.0e38], np.float32)
    bits = W.to_bf16_bits(x)
    back = W.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to even (1.0); 1 + 3*2^-8 rounds up to 1 + 2^-6
    np.testing.assert_array_equal(back[:6], np.array([1.0, 1.0, 1.0 + 2**-7, 1.0 + 2**-6, -2.5, 0.0], np.float32))
    import torch
    y = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(W.to_bf16_bits(y), ref)


def test_determinism_and_chunked_draws():
    a = W.draw(T=100, V=70000, D=16, K=4, seed=3, ids="zipf", mask="random", mask_frac=0.1)
    b = W.draw(T=100, V=70000, D=16, K=4, seed=3, ids="zipf", mask="random", mask_frac=0.1)
    for f in ("H", "E", "targets", "mask"):
        np.testing.assert_array_equal(getattr(a, f), getattr(b, f))
    # the chunked row draws equal one big draw from the same stream
    g1 = np.random.Generator(np.random.PCG64(np.random.SeedSequence(3).spawn(5)[1]))
    big = g1.standard_normal((70000, 16), dtype=np.float32) * np.float32(1 / np.sqrt(16))
    np.testing.assert_array_equal(W.bf16_bits_to_f32(W.to_bf16_bits(big)), a.E)


@pytest.mark.parametrize("name", ["tiny_f32", "small_catalog"])
def test_config_recipes(name):
    p = W.draw_config(name)
    cfg = W.CONFIGS[name]
    assert p.H.shape == (cfg["T"], cfg["D"]) and p.E.shape == (cfg["V"], cfg["D"])
    assert p.targets.shape == (cfg["T"], cfg["K"]) and p.targets.dtype == np.int32
    for row in p.targets:
        ids = row[row >= 0]
        assert len(np.unique(ids)) == len(ids)
        assert np.all(row[len(ids):] == -1)
        assert np.all((ids >= 0) & (ids < cfg["V"]))
    if name == "tiny_f32":
        assert p.dtype == "f32" and p.H_bits is None
        assert int((p.mask == 0).sum()) == round(0.1 * 64)
        assert np.all((p.targets >= 0).sum(1) == 4)
    else:
        assert np.all(p.mask.reshape(32, 200)[:, 170:] == 0) and np.all(p.mask.reshape(32, 200)[:, :170] == 1)
        np.testing.assert_array_equal(W.bf16_bits_to_f32(p.H_bits), p.H)
        # bounded Zipf: item 0 is the most frequent id
        counts = np.bincount(p.targets[p.targets >= 0], minlength=p.V)
        assert counts.argmax() == 0 and counts[0] > 0.05 * (p.targets >= 0).sum()
        assert abs(p.E.std() - 1 / 8) < 0.01 and abs(p.H.std() - 1.0) < 0.05


def test_poisson_counts_clip():
    p = W.draw(T=3000, V=5000, D=8, K=16, count="poisson", count_mean=3.0, count_max=16,
               ids="zipf", zipf_s=1.05, mask="trailing", B=15, N=200, trailing=40)
    c = (p.targets >= 0).sum(1)
    assert c.min() >= 1 and c.max() <= 16
    assert abs(c.mean() - 3.0) < 0.2
    assert (p.mask == 0).sum() == 15 * 40
