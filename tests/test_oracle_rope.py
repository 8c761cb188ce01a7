"""Pins of the oracle's fused RoPE + Smooth-QK + quantise path: rotate-half RoPE in fp32
(each product and the sum rounded once) from a caller-supplied angle table, followed by
the same Smooth-QK scaling and 4-bit quantiser as the unfused path."""
import numpy as np

from bit_flashattention_b200 import gen


def _bf16(rng, shape, scale=1.0):
    return gen.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _table(N, d, theta=1e4, pos0=0):
    inv = theta ** (-np.arange(0, d // 2, dtype=np.float64) * 2.0 / d)
    ang = (pos0 + np.arange(N, dtype=np.float64))[:, None] * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def test_position_zero_is_identity(orc):
    rng = np.random.default_rng(21)
    x = _bf16(rng, (1, 2, 4, 64))
    cos, sin = _table(4, 64)
    out = orc.rope_rows(x, cos, sin)
    assert np.array_equal(out[:, :, 0, :], gen.bf16_bits_to_f32(x)[:, :, 0, :])


def test_quarter_turn_is_exact_rotate_half(orc):
    # cos = 0, sin = 1 everywhere: (x1, x2) -> (-x2, x1) for the pair (i, i + d/2)
    rng = np.random.default_rng(22)
    x = _bf16(rng, (1, 1, 8, 128))
    cos = np.zeros((8, 64), np.float32)
    sin = np.ones((8, 64), np.float32)
    out = orc.rope_rows(x, cos, sin)
    xf = gen.bf16_bits_to_f32(x)
    assert np.array_equal(out[..., :64], -xf[..., 64:])
    assert np.array_equal(out[..., 64:], xf[..., :64])


def test_matches_float64_rotation_within_rounding(orc):
    rng = np.random.default_rng(23)
    N, d = 300, 128
    x = _bf16(rng, (2, 3, N, d), scale=4.0)
    cos, sin = _table(N, d, theta=1e6, pos0=17)
    out = orc.rope_rows(x, cos, sin).astype(np.float64)
    xf = gen.bf16_bits_to_f32(x).astype(np.float64)
    c, s = cos.astype(np.float64), sin.astype(np.float64)
    x1, x2 = xf[..., :64], xf[..., 64:]
    ref = np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)
    mag = np.concatenate([np.abs(x1 * c) + np.abs(x2 * s), np.abs(x2 * c) + np.abs(x1 * s)], axis=-1)
    # two rounded products and one rounded sum: |err| <= 2^-24 (|a| + |b|) + 2^-24 |result|
    bound = 2.0 ** -24 * (mag + np.abs(ref)) * 1.0001 + 1e-45
    assert np.all(np.abs(out - ref) <= bound)
    # the rotation keeps every pair's norm (to rounding)
    n_in = x1 ** 2 + x2 ** 2
    n_out = out[..., :64] ** 2 + out[..., 64:] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-6, atol=1e-30)


def test_fused_equals_unfused_when_the_rotation_is_exact(orc):
    # angles that are multiples of 90 degrees make every rotated value a bf16 value, so
    # RoPE-then-quantise (fused) must equal quantising the rotated bf16 tensor (unfused),
    # with and without Smooth-QK scales
    rng = np.random.default_rng(24)
    B, H, Hkv, N, d = 1, 4, 2, 32, 128
    x = _bf16(rng, (B, H, N, d))
    quarter = rng.integers(0, 4, (N, d // 2))
    cos = np.choose(quarter, [1.0, 0.0, -1.0, 0.0]).astype(np.float32)
    sin = np.choose(quarter, [0.0, 1.0, 0.0, -1.0]).astype(np.float32)
    xf = gen.bf16_bits_to_f32(x)
    x1, x2 = xf[..., : d // 2], xf[..., d // 2:]
    rotated = np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1).astype(np.float32)
    rot_bits = gen.f32_to_bf16_bits(rotated)
    assert np.array_equal(gen.bf16_bits_to_f32(rot_bits), rotated)
    s = np.exp2(rng.integers(-3, 4, (Hkv, d))).astype(np.float32) * np.float32(1.25)
    for scale in (None, s):
        fc, fs = orc.quantize_rows_rope(x, Hkv, cos, sin, scale)
        uc, us = orc.quantize_rows(rot_bits, Hkv, scale)
        assert np.array_equal(fc, uc) and np.array_equal(fs, us)


def test_exact_cancellation_is_positive_zero(orc):
    # equal and opposite rounded products sum to +0 (round to nearest)
    x = np.array([[[[1.5, -2.25, -1.5, 2.25]]]], np.float32)      # d = 4: pairs (0, 2), (1, 3)
    bits = gen.f32_to_bf16_bits(x)
    cos = np.full((1, 2), 0.5, np.float32)
    sin = np.full((1, 2), 0.5, np.float32)
    out = orc.rope_rows(bits, cos, sin)
    assert np.array_equal(out[..., 2:], np.zeros((1, 1, 1, 2), np.float32))
    assert not np.any(np.signbit(out[..., 2:]))
