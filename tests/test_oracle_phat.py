"""Pins of the oracle's P_hat evaluation: P / sigma computed in the log domain,
y = p(frac(128u)) * 2^(floor(128u) - 125) with u = sat(S*c/128 + B) and
B = (L(sigma) - m + 125) / 128, L(sigma) = RN(-log2 sigma)."""
import ml_dtypes
import numpy as np


def _e4m3(code):
    return float(np.array([code], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)[0])


def test_neg_log2_scale_is_rounded_log(orc):
    for code in range(1, 0x7F):
        sig = _e4m3(code)
        L = orc.neg_log2_scale(code)
        ref = -np.log2(sig)
        assert abs(L - ref) <= 0.5 * np.spacing(np.float32(abs(ref))) + 1e-12, (code, L, ref)


def _bias(L, m):
    a = np.float32(np.float32(L) - np.float32(m))
    return np.float32(np.float32(a + np.float32(125.0)) * np.float32(0.0078125))


def test_phat_value_is_p_over_sigma(orc):
    rng = np.random.default_rng(13)
    c = np.float32(1.4426950408889634 / np.sqrt(128.0))
    for code in (0x08, 0x20, 0x2C, 0x30, 0x33, 0x38, 0x40, 0x55):
        sig = _e4m3(code)
        m = np.float32(rng.uniform(-5, 30))
        S = ((m + rng.uniform(-12, 0.01, 20000)) / c).astype(np.float32)
        y = orc.phat_values(S, c, _bias(orc.neg_log2_scale(code), m)).astype(np.float64)
        ref = np.exp2(S.astype(np.float64) * float(c) - float(m)) / sig
        live = (ref > 2.0 ** -100) & (ref < 7.9)
        assert np.max(np.abs(y[live] / ref[live] - 1)) <= 2.2e-3


def test_phat_value_saturates_at_both_ends(orc):
    c = np.float32(0.125)
    B = _bias(orc.neg_log2_scale(0x38), 0.0)               # sigma = 1, m = 0
    y = orc.phat_values(np.array([-np.inf, -1e6, 1e6, 0.0], np.float32), c, B)
    assert y[0] == 2.0 ** -125 and y[1] == 2.0 ** -125       # u clamped to 0
    assert y[2] == 8.0                                       # u clamped to 1: code 7 (6.0) anyway
    assert y[3] == np.float32(1.0)                           # P = 1, sigma = 1
    yz = orc.phat_values(np.array([0.0, 5.0], np.float32), c, np.float32(-np.inf))
    assert np.all(yz == 2.0 ** -125)                         # sigma == 0: every code 0


def test_codes_match_direct_product_away_from_boundaries(orc):
    # The E2M1 codes of y agree with the codes of E(S c - m) * RN(1/sigma) except where the
    # two evaluations straddle a rounding boundary (both approximate the same P/sigma).
    rng = np.random.default_rng(14)
    c = np.float32(1.4426950408889634 / np.sqrt(128.0))
    m = np.float32(3.0)
    S = ((m + rng.uniform(-8, 0, 200000)) / c).astype(np.float32)
    code = 0x2E
    sig = np.float32(_e4m3(code))
    y_new = orc.phat_values(S, c, _bias(orc.neg_log2_scale(code), m))
    y_old = orc.exp2((S * c).astype(np.float32) - m) * (np.float32(1.0) / sig)
    c_new, c_old = orc.e2m1_encode(y_new), orc.e2m1_encode(y_old)
    assert np.mean(c_new != c_old) < 5e-3
