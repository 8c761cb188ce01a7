"""Pins of the oracle's P_hat code decision: the E2M1 code of y, where y is P / sigma
evaluated in the log domain with a linear mantissa,
u = sat(S*c/128 + B), B = (L(sigma) - m + 125) / 128, L(sigma) = RN(-log2 sigma),
z = 128u - 125 + delta (on a 2^-10 grid), y = 2^floor(z) * (1 + frac z).

The pins compare against the exact value r = 2^(S c - m) / sigma computed in float64 and
rounded to E2M1 by ml_dtypes: the codes agree wherever r is not within the stated
distance of an E2M1 rounding boundary, the boundaries themselves sit within that distance
of the exact ones, and y stays within the linear-mantissa band around r."""
import ml_dtypes
import numpy as np

# E2M1 rounding boundaries (round to nearest, ties to even) between consecutive codes
BOUNDS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
NEAR = 0.0145          # log2 distance for every boundary but the lowest
NEAR_LOW = (-0.001, 0.0725)   # the 0.25 boundary is shifted up by about 0.071


def _e4m3(code):
    return float(np.array([code], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)[0])


def _e2m1_codes(x):
    """E2M1 codes (0..7) of non-negative values, by ml_dtypes (RN, ties to even, saturating)."""
    v = np.minimum(np.asarray(x, np.float64), 6.0).astype(ml_dtypes.float4_e2m1fn)
    return np.asarray(v).view(np.uint8) & 0x7


def _bias(L, m):
    a = np.float32(np.float32(L) - np.float32(m))
    return np.float32(np.float32(a + np.float32(125.0)) * np.float32(0.0078125))


def _far_from_bounds(lr):
    far = np.ones(lr.shape, bool)
    for t in BOUNDS[1:]:
        far &= np.abs(lr - np.log2(t)) > NEAR
    d0 = lr + 2.0
    far &= ~((d0 > NEAR_LOW[0]) & (d0 < NEAR_LOW[1]))
    return far


def test_neg_log2_scale_is_rounded_log(orc):
    for code in range(1, 0x7F):
        sig = _e4m3(code)
        L = orc.neg_log2_scale(code)
        ref = -np.log2(sig)
        assert abs(L - ref) <= 0.5 * np.spacing(np.float32(abs(ref))) + 1e-12, (code, L, ref)


def test_codes_equal_exact_codes_away_from_boundaries(orc):
    rng = np.random.default_rng(13)
    c = np.float32(1.4426950408889634 / np.sqrt(128.0))
    n_far = n_all = 0
    for code in (0x08, 0x20, 0x2C, 0x30, 0x33, 0x38, 0x40, 0x55):
        sig = _e4m3(code)
        m = np.float32(rng.uniform(-5, 30))
        # log2(P / sigma) spread over the codes' range and a little beyond
        lr_target = rng.uniform(-4.0, 3.5, 40000)
        S = ((lr_target + np.log2(sig) + float(m)) / float(c)).astype(np.float32)
        y = orc.phat_values(S, c, _bias(orc.neg_log2_scale(code), m))
        lr = S.astype(np.float64) * float(c) - float(m) - np.log2(sig)
        far = _far_from_bounds(lr)
        got = orc.e2m1_encode(y) & 0x7
        want = _e2m1_codes(np.exp2(lr))
        assert np.array_equal(got[far], want[far]), (code, np.flatnonzero(got[far] != want[far])[:5])
        n_far += int(far.sum())
        n_all += far.size
    assert n_far > 0.9 * n_all


def test_boundaries_lie_near_the_exact_ones(orc):
    # sigma = 1, m = 0: scan log2(P / sigma) across each boundary on a fine grid
    c = np.float32(0.125)
    B = _bias(orc.neg_log2_scale(0x38), 0.0)
    for t in BOUNDS:
        lo, hi = np.log2(t) - 0.1, np.log2(t) + 0.1
        S = np.arange(lo / 0.125, hi / 0.125, 2.0 ** -14, dtype=np.float64).astype(np.float32)
        codes = orc.e2m1_encode(orc.phat_values(S, c, B)) & 0x7
        assert np.all(np.diff(codes.astype(int)) >= 0)                 # monotone in S
        k = int(np.argmax(codes > codes[0]))
        assert k > 0 and codes[k] == codes[0] + 1
        where = float(S[k]) * 0.125 - np.log2(t)                       # boundary offset, log2 units
        if t == 0.25:
            assert NEAR_LOW[0] < where < NEAR_LOW[1], (t, where)
            assert where > 0.06                                        # shifted up, not down
        else:
            assert abs(where) < NEAR, (t, where)


def test_value_stays_in_the_linear_mantissa_band(orc):
    # y / (P / sigma) = (1 + f) 2^(delta - f), f = frac(z): between 2^delta and 1.0615 * 2^delta
    rng = np.random.default_rng(15)
    c = np.float32(1.4426950408889634 / np.sqrt(128.0))
    for code in (0x20, 0x38, 0x4E):
        sig = _e4m3(code)
        m = np.float32(rng.uniform(0, 20))
        S = ((m + rng.uniform(-20, 2.5, 50000) + np.log2(sig)) / c).astype(np.float32)
        y = orc.phat_values(S, c, _bias(orc.neg_log2_scale(code), m)).astype(np.float64)
        ref = np.exp2(S.astype(np.float64) * float(c) - float(m)) / sig
        q = y / ref
        assert q.min() > 0.9510 and q.max() < 1.0107, (q.min(), q.max())


def test_value_saturates_at_both_ends(orc):
    c = np.float32(0.125)
    B = _bias(orc.neg_log2_scale(0x38), 0.0)                 # sigma = 1, m = 0
    S = np.array([-np.inf, -1e6, 1e6, np.inf, np.nan], np.float32)
    codes = orc.e2m1_encode(orc.phat_values(S, c, B)) & 0x7
    assert list(codes) == [0, 0, 7, 7, 0]                     # u clamped to [0, 1]; NaN -> 0
    y = orc.phat_values(S[:1], c, B)
    assert 0.0 < y[0] < 2.0 ** -124                           # still a normal float
    yz = orc.phat_values(np.array([0.0, 5.0, 1e6], np.float32), c, np.float32(-np.inf))
    assert np.all(orc.e2m1_encode(yz) & 0x7 == 0)             # sigma == 0: every code 0
