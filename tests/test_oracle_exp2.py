"""Pins of the method's own exp2 approximation E(x) used for the softmax weights.

E(x) = p(f) * 2^n with n = floor(max(x, -127)), f = RN(x - n) and p a cubic with p(0) = 1;
its properties are pinned against numpy's exp2 (a library routine) and closed forms.
The bound 9e-5 is the one a cubic fit of 2^f on [0, 1) reaches; a quadratic (about 2e-3)
or a wrong coefficient fails it.
"""
import numpy as np


def _all_f32_in(lo_bits, hi_bits):
    return np.arange(lo_bits, hi_bits, dtype=np.uint32).view(np.float32)


def test_relative_error_bound_exhaustive_one_octave(orc):
    # every fp32 in [-2, -1): f runs over [0, 1) at full resolution
    x = _all_f32_in(0xBF800000, 0xC0000000)
    e = orc.exp2(x).astype(np.float64)
    rel = np.abs(e / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() <= 9e-5


def test_relative_error_bound_sampled_range(orc):
    rng = np.random.default_rng(3)
    x = rng.uniform(-126, 0.5, 2_000_000).astype(np.float32)
    e = orc.exp2(x).astype(np.float64)
    assert np.max(np.abs(e / np.exp2(x.astype(np.float64)) - 1)) <= 9e-5


def test_integers_exact_and_underflow(orc):
    k = np.arange(-126, 1, dtype=np.float32)
    assert np.array_equal(orc.exp2(k), np.exp2(k.astype(np.float64)).astype(np.float32))
    x = np.array([-127.0, -200.0, -np.inf, -1e30, np.nan], np.float32)
    assert np.all(orc.exp2(x) == 0.0)


def test_polynomial_monotone_over_every_fp32_fraction(orc):
    # For x in [0, 1), n = 0 and E(x) = p(x): this walks p over every fp32 f in [0, 1).
    # With p(1) <= 2 (next test) that makes E monotone on its whole domain, so the block
    # maximum of P is E of the block maximum of the exponent arguments.
    prev = -np.inf
    step = 1 << 25
    for lo in range(0x00000000, 0x3F800000, step):
        x = _all_f32_in(lo, min(lo + step, 0x3F800000))
        e = orc.exp2(x)
        assert e[0] >= prev
        assert np.all(e[1:] >= e[:-1]), hex(lo)
        prev = e[-1]


def test_fraction_rounding_up_to_one_stays_below_the_next_power(orc):
    # x just below an integer n + 1 can give f = RN(x - n) = 1.0: E must not pass 2^(n+1)
    for n in (-126, -60, -3, -1):
        x = np.nextafter(np.float32(n + 1), np.float32(-1e9), dtype=np.float32)
        xs = np.array([x - np.float32(i) * abs(np.spacing(x)) for i in range(64)], np.float32)
        assert np.all(orc.exp2(xs) <= np.float32(2.0) ** (n + 1))
    tiny = -np.float32(2.0) ** -np.arange(25, 60).astype(np.float32)
    assert np.all(orc.exp2(tiny) <= 1.0)


def test_monotone_around_every_integer(orc):
    # exhaustive over [-2, -0.5] plus every integer boundary in [-126, 0]
    x = _all_f32_in(0xBF000000, 0xC0000001)[::-1]                       # -2 .. -0.5, increasing
    e = orc.exp2(x)
    assert np.all(np.diff(e.astype(np.float64)) >= 0)
    for n in range(-126, 1):
        b = np.float32(n).view(np.uint32).astype(np.int64)
        around = np.sort((b + np.arange(-300, 301)).astype(np.uint32).view(np.float32))
        around = around[(around >= -126.5) & (around <= 0.5)]
        assert np.all(np.diff(orc.exp2(np.sort(around)).astype(np.float64)) >= 0)
