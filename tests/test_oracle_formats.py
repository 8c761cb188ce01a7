"""Pins of the oracle's 4-bit/8-bit format rules against library conversions and the
format definitions (not against the oracle itself).

The 4-bit format is the one the HiFA4 abstract leaves open ("HIF4"); the reading used
here is NVFP4-style: E2M1 codes with one unsigned E4M3 scale per 16 elements.
"""
import ml_dtypes
import numpy as np
import torch


def _boundary_values():
    """fp32 values around every E2M1 midpoint and value, plus a random spread."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)
    out = [mids]
    for m in mids:
        u = np.float32(m).view(np.uint32).astype(np.int64)
        out.append((u + np.arange(-64, 65)).astype(np.uint32).view(np.float32))
    rng = np.random.default_rng(1)
    out.append(rng.uniform(-8, 8, 200000).astype(np.float32))
    out.append((rng.standard_normal(200000) * 10.0 ** rng.uniform(-4, 2, 200000)).astype(np.float32))
    out.append(np.array([0.0, -0.0, 7.0, 1e30, -1e30, np.inf, -np.inf, 1e-40, -1e-40], np.float32))
    v = np.concatenate(out)
    return np.concatenate([v, -v])


def test_e2m1_encode_matches_ml_dtypes(orc):
    x = _boundary_values()
    got = orc.e2m1_encode(x)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(got, ref)


def test_e2m1_values_from_definition(orc):
    # E2M1: sign s, exponent e (2 bits, bias 1), mantissa m (1 bit);
    # e == 0 -> m * 0.5 (subnormal), else 2^(e-1) * (1 + m/2).
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        v = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
        assert orc.e2m1_value(code) == (-v if s else v)


def test_e4m3_values_from_definition(orc):
    # E4M3 (OCP FP8): bias 7, e == 0 -> m/8 * 2^-6, else (1 + m/8) * 2^(e-7); 0x7F is NaN.
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        v = (m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        assert orc.e4m3_value(code) == v
    assert orc.e4m3_value(0x7E) == 448.0


def test_e4m3_encode_matches_torch_cast(orc):
    rng = np.random.default_rng(2)
    x = np.concatenate([
        (10.0 ** rng.uniform(-5, 2.66, 400000)).astype(np.float32),
        np.array([orc.e4m3_value(c) for c in range(0x7F)], np.float32),
    ])
    # every midpoint between neighbouring codes (ties go to even)
    vals = np.array([orc.e4m3_value(c) for c in range(0x7F)], np.float64)
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    near = np.concatenate([(mids.view(np.uint32).astype(np.int64) + k).astype(np.uint32).view(np.float32)
                           for k in (-2, -1, 0, 1, 2)])
    x = np.concatenate([x, near])
    x = x[(x > 0) & (x < 464.0)]       # torch's cast turns >= 464 into NaN instead of saturating
    got = orc.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)
    ref2 = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(got, ref2)


def test_e4m3_encode_saturates_and_zero(orc):
    x = np.array([464.0, 480.0, 1e6, np.inf, 0.0, -0.0, 2.0 ** -10, 2.0 ** -11], np.float32)
    got = orc.e4m3_encode(x)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0, 0, 0, 0]   # 2^-10 is the 0 / 2^-9 tie -> even (0)
