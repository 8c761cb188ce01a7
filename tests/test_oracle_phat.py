"""Pins of the oracle's P -> P_hat step: each 16 consecutive keys of a row's P form one
block of the 4-bit format, so P_hat must be the round-to-nearest of P on its block's grid
{0, 0.5, 1, 1.5, 2, 3, 4, 6} x sigma, with sigma the E4M3 value nearest to the block's
largest P divided by 6.

The pins check those properties against facts that do not come from the oracle's own
formula: the E2M1 and E4M3 value sets decoded by ml_dtypes, the definition of rounding to
nearest (no grid point closer than the chosen one), the top code of a block, and float64
ratios.  A rounding shortcut that moves the code boundaries (a linear-mantissa exponential,
a shifted boundary, a truncation) fails the nearest-grid-point pin on a few percent of the
scores; a block scale taken from the wrong maximum fails the scale pin."""
import ml_dtypes
import numpy as np

from bit_flashattention_b200 import gen

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
E4M3 = np.arange(0, 0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)   # codes 0..126


def _qwen_like_rows(orc, seed=71, causal=True):
    """A small causal GQA case with Qwen-sized heads (d = 128, 128-key tiles), K outlier
    channels and Smooth-QK: scores spread over many log2 units."""
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, N, d = 1, 2, 1, 512, 128
    q = rng.standard_normal((B, Hq, N, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    k[..., rng.choice(d, 8, replace=False)] *= 10.0
    k += rng.standard_normal((1, Hkv, 1, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    q, k, v = (gen.f32_to_bf16_bits(a) for a in (q, k, v))
    s, sinv = orc.calibrate(q, k, 0.5)
    return orc.quantize_all(q, k, v, s, sinv), causal


def _blocks(orc, qz, causal, bc, rows):
    """(P, P_hat) of every visited 16-key block of the given rows, [n, 16] float64 each."""
    P, Ph = [], []
    for r in rows:
        tr = orc.attn_trace(qz, causal, bc, int(r))
        P.append(tr["p"].astype(np.float64).reshape(-1, 16))
        Ph.append(tr["phat"].astype(np.float64).reshape(-1, 16))
    return np.concatenate(P), np.concatenate(Ph)


def _sigma_nearest(amax):
    """The E4M3 value(s) nearest to amax / 6 (both neighbours on an exact tie)."""
    t = amax / 6.0
    dist = np.abs(E4M3[None, :] - t[:, None])
    return dist, dist.min(1)


def test_block_scale_is_the_e4m3_value_nearest_to_amax_over_six(orc):
    qz, causal = _qwen_like_rows(orc)
    P, Ph = _blocks(orc, qz, causal, 128, range(5, qz.Hq * qz.N, 41))
    amax = P.max(1)
    live = Ph.max(1) > 0
    # the block's largest P gets its largest P_hat, and every P_hat is code * sigma with
    # sigma = P_hat_max / 6 when the top code is 6 (it is, whenever sigma is normal)
    sigma = Ph.max(1) / 6.0
    normal = live & (sigma >= 2.0 ** -6)
    assert normal.sum() > 100
    top = np.argmax(P, 1)
    assert np.array_equal(Ph[np.arange(len(P)), top][live], Ph.max(1)[live])
    dist, best = _sigma_nearest(amax[normal])
    got = np.abs(sigma[normal] - amax[normal] / 6.0)
    # RN(amax * RN(1/6)) differs from amax/6 by < 2 ulps of fp32: allow that slack
    assert np.all(got <= best + 4 * 2.0 ** -24 * amax[normal] / 6.0)
    # blocks whose amax / 6 is below half the smallest E4M3 step (2^-10) are flushed
    assert np.all(Ph[amax / 6.0 < 2.0 ** -10 * 0.99] == 0.0)


def test_phat_is_a_nearest_grid_point_of_p(orc):
    qz, causal = _qwen_like_rows(orc)
    P, Ph = _blocks(orc, qz, causal, 128, range(0, qz.Hq * qz.N))
    sigma = Ph.max(1) / 6.0
    blocks = (sigma >= 2.0 ** -6)                     # a normal scale: the top code is 6
    P, Ph, sigma = P[blocks], Ph[blocks], sigma[blocks]
    r = P / sigma[:, None]                            # exact P / sigma in float64
    code = Ph / sigma[:, None]
    assert np.all(np.isin(code, E2M1))
    rs = np.minimum(r, 6.0)                           # satfinite: everything above 6 is 6
    err = np.abs(code - rs)
    best = np.abs(E2M1[None, None, :] - rs[..., None]).min(-1)
    # the chosen value is a nearest one; a difference can only come from the one fp32
    # rounding of P * RN(1/sigma) at an exact midpoint (relative 2^-23 of r)
    slack = 2.0 ** -22 * np.maximum(r, 1.0)
    bad = err > best + slack
    assert r.size > 20000 and not bad.any(), (bad.sum(), r[bad][:5], code[bad][:5])
    # and the test is sensitive: a fair share of scores lies in every code's interval
    for c in E2M1[1:]:
        assert np.count_nonzero(code == c) > 200, c


def test_phat_error_bound(orc):
    qz, causal = _qwen_like_rows(orc, seed=72, causal=False)
    P, Ph = _blocks(orc, qz, causal, 128, range(1, qz.Hq * qz.N, 53))
    sigma = Ph.max(1) / 6.0
    live = sigma >= 2.0 ** -6                         # a normal scale: the top code is 6
    # |P_hat - P| <= half the local spacing of the grid: 0.25 sigma below 2 sigma, 0.5
    # sigma up to 4 sigma, 1 sigma up to 6 sigma
    r = P[live] / sigma[live, None]
    half = np.where(r < 2.0, 0.25, np.where(r < 4.0, 0.5, 1.0))
    assert np.all(np.abs(Ph[live] / sigma[live, None] - np.minimum(r, 6.0)) <= half * (1 + 2.0 ** -20))


def test_zero_and_masked_keys_give_zero(orc):
    qz, _ = _qwen_like_rows(orc)
    # causal row 130 of head 0: tile 1 (keys 128..255) holds keys 131..255, all masked
    tr = orc.attn_trace(qz, True, 128, 130)
    assert np.all(tr["p"][1, 3:] == 0.0) and np.all(tr["phat"][1, 3:] == 0.0)
    assert tr["phat"][1, :3].max() > 0.0
