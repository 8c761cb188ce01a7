"""Pins of the method's own exp2 approximation E(x) used for the softmax weights.

E(x) = p(f) * 2^n with n = floor(max(x, -127)), f = x - n and p a quadratic with p(0) = 1;
its properties are pinned against numpy's exp2 (a library routine) and closed forms.
"""
import numpy as np


def _all_f32_in(lo_bits, hi_bits):
    return np.arange(lo_bits, hi_bits, dtype=np.uint32).view(np.float32)


def test_relative_error_bound_exhaustive_one_octave(orc):
    # every fp32 in [-2, -1): f runs over [0, 1) at full resolution
    x = _all_f32_in(0xBF800000, 0xC0000000)
    e = orc.exp2(x).astype(np.float64)
    rel = np.abs(e / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() <= 2.1e-3


def test_relative_error_bound_sampled_range(orc):
    rng = np.random.default_rng(3)
    x = rng.uniform(-126, 0.5, 2_000_000).astype(np.float32)
    e = orc.exp2(x).astype(np.float64)
    assert np.max(np.abs(e / np.exp2(x.astype(np.float64)) - 1)) <= 2.1e-3


def test_integers_exact_and_underflow(orc):
    k = np.arange(-126, 1, dtype=np.float32)
    assert np.array_equal(orc.exp2(k), np.exp2(k.astype(np.float64)).astype(np.float32))
    x = np.array([-127.0, -200.0, -np.inf, -1e30, np.nan], np.float32)
    assert np.all(orc.exp2(x) == 0.0)


def test_monotone_non_decreasing(orc):
    # exhaustive over [-2, -0.5] plus every integer boundary in [-126, 0]
    x = _all_f32_in(0xBF000000, 0xC0000001)[::-1]                       # -2 .. -0.5, increasing
    e = orc.exp2(x)
    assert np.all(np.diff(e.astype(np.float64)) >= 0)
    for n in range(-126, 1):
        b = np.float32(n).view(np.uint32).astype(np.int64)
        around = np.sort((b + np.arange(-300, 301)).astype(np.uint32).view(np.float32))
        around = around[(around >= -126.5) & (around <= 0.5)]
        assert np.all(np.diff(orc.exp2(np.sort(around)).astype(np.float64)) >= 0)
