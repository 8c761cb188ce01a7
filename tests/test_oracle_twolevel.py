"""Pins of the oracle's two-level P scale (an ablation variant of the 4-bit format: a
per-row, per-tile power of two 2^k under the E4M3 block scales of P).  It must give the
one-level results exactly where every block scale of P is a normal E4M3 value, keep every
element within the E2M1 rounding bound of its block far below the range where one level
flushes blocks to zero, and so lose less probability mass."""
import numpy as np

from bit_flashattention_b200 import gen


def _bf16(rng, shape, scale):
    return gen.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _inputs(orc, rng, B, Hq, Hkv, N, d, qk_scale):
    q = _bf16(rng, (B, Hq, N, d), qk_scale)
    k = _bf16(rng, (B, Hkv, N, d), qk_scale)
    v = _bf16(rng, (B, Hkv, N, d), 1.0)
    return orc.quantize_all(q, k, v), (q, k, v)


def _block_amax(p):
    """[tiles, bc] unquantised P -> [tiles, bc/16] block maxima."""
    return p.reshape(p.shape[0], -1, 16).max(-1)


def test_equals_one_level_when_every_block_scale_is_normal(orc):
    # small scores: every block amax of P stays above 6 * 2^-6, so each one-level scale
    # E4M3(amax/6) is normal and E4M3 rounding commutes with the power of two 2^-k
    rng = np.random.default_rng(61)
    B, Hq, Hkv, N, d, bc = 1, 2, 1, 256, 64, 64
    qz, _ = _inputs(orc, rng, B, Hq, Hkv, N, d, 0.3)
    for causal in (False, True):
        rows = np.arange(B * Hq * N, dtype=np.int64)
        one = orc.attn_fwd(qz, causal, bc, rows)
        two = orc.attn_fwd(qz, causal, bc, rows, two_level=True)
        for r in range(0, B * Hq * N, 7):
            tr = orc.attn_trace(qz, causal, bc, r)
            am = _block_amax(tr["p"])
            visible = am > 2.0 ** -100                         # blocks with an unmasked key
            assert np.all(am[visible] >= 6 * 2.0 ** -6), r
            tr2 = orc.attn_trace(qz, causal, bc, r, two_level=True)
            assert np.array_equal(tr["phat"], tr2["phat"])
        assert np.array_equal(one["o_bf16"], two["o_bf16"])
        assert np.array_equal(one["m"], two["m"]) and np.array_equal(one["l"], two["l"])


def _spread_rows(orc, seed=62):
    # large scores: most keys sit many log2 units below the row maximum, so many blocks
    # of P are far below 6 * 2^-10 (one-level scale 0) or in the E4M3 subnormal range
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, N, d, bc = 1, 2, 1, 512, 128, 128
    qz, raw = _inputs(orc, rng, B, Hq, Hkv, N, d, 2.2)
    return qz, raw, bc


def test_elements_within_the_e2m1_bound_of_their_block(orc):
    qz, _, bc = _spread_rows(orc)
    n_small_kept = 0
    for r in range(3, qz.Hq * qz.N, 37):
        one = orc.attn_trace(qz, False, bc, r)
        two = orc.attn_trace(qz, False, bc, r, two_level=True)
        p, ph1, ph2 = one["p"].astype(np.float64), one["phat"].astype(np.float64), two["phat"].astype(np.float64)
        assert np.array_equal(p, two["p"])
        am = _block_amax(one["p"]).astype(np.float64)
        e_t = np.floor(np.log2(am.max(1, keepdims=True)))
        # the block scale is E4M3(amax/6 * 2^-k) * 2^k with 2^k = 2^(e_t - 10): within 1/16
        # of amax / 6 when normal, within half the subnormal step 2^(k - 9) otherwise
        sig_hi = np.repeat(am / 6.0 * 1.0625 + 2.0 ** (e_t - 20), 16, axis=1)
        # E2M1 of x = P / sigma: relative error <= 0.36 for x >= 0.5 (the 0.75 boundary, moved
        # by the log-domain rule), absolute <= 0.2625 sigma below (the 0.25 boundary moved by
        # 0.071 log2 units)
        bound = np.maximum(0.36 * p, 0.2625 * sig_hi)
        kept = np.repeat(am / 6.0 > 2.0 ** (e_t - 20) * 1.01, 16, axis=1)
        assert np.all((np.abs(ph2 - p) <= bound)[kept]), r
        assert np.all(ph2 <= 6.0 * sig_hi) and np.all(ph2 >= 0.0)
        # the scale survives exactly when amax/6 * 2^-k lies above 2^-10 (half the smallest
        # E4M3 step): the block's largest element keeps a non-zero code, below it all are 0
        gone = np.repeat(am / 6.0 < 2.0 ** (e_t - 20) / 1.01, 16, axis=1)
        assert np.all(ph2[gone] == 0.0)
        top = (p == np.repeat(am, 16, axis=1)) & kept
        assert np.all(ph2[top] > 0.0)
        # one level flushes blocks with amax <= 6 * 2^-10 to zero
        flushed = np.repeat(am <= 6 * 2.0 ** -10, 16, axis=1)
        assert np.all(ph1[flushed] == 0.0)
        n_small_kept += int(np.sum((ph2 > 0) & flushed))
    assert n_small_kept > 100


def test_less_probability_mass_lost(orc):
    # eps = sum P_hat / sum P - 1 per tile: one level loses the mass of the flushed and
    # subnormal-scale blocks; the two-level scale keeps it to the E2M1 rounding bias
    qz, _, bc = _spread_rows(orc, seed=63)
    e1, e2 = [], []
    for r in range(5, qz.Hq * qz.N, 29):
        one = orc.attn_trace(qz, False, bc, r)
        two = orc.attn_trace(qz, False, bc, r, two_level=True)
        sp = one["p"].astype(np.float64).sum(1)
        e1.append(one["phat"].astype(np.float64).sum(1) / sp - 1.0)
        e2.append(two["phat"].astype(np.float64).sum(1) / sp - 1.0)
    e1, e2 = np.concatenate(e1), np.concatenate(e2)
    print(f"\nmean eps per tile: one level {np.mean(e1):.4f}, two-level {np.mean(e2):.4f}")
    assert np.mean(e1) < -0.05
    assert abs(np.mean(e2)) < 0.5 * abs(np.mean(e1))
    assert np.mean(np.abs(e2)) < np.mean(np.abs(e1))


def test_closer_to_exact_attention(orc):
    # fp64 softmax attention on the same dequantised Q, K, V: the two-level output is at
    # least as close as the one-level output on score-spread inputs
    from tests.test_oracle_quant import _dequant
    qz, _, bc = _spread_rows(orc, seed=64)
    rows = np.arange(0, qz.Hq * qz.N, dtype=np.int64)
    one = orc.attn_fwd(qz, False, bc, rows, want_f64=True)["o_f64"]
    two = orc.attn_fwd(qz, False, bc, rows, want_f64=True, two_level=True)["o_f64"]
    qd = _dequant(qz.qc, qz.qs)[0].astype(np.float64)
    kd = _dequant(qz.kc, qz.ks)[0].astype(np.float64)
    vd = _dequant(qz.vc, qz.vs)[0].astype(np.float64).swapaxes(-1, -2)      # [Hkv, N, d]
    ref = []
    for h in range(qz.Hq):
        S = qd[h] @ kd[0].T / np.sqrt(qz.d)
        P = np.exp(S - S.max(1, keepdims=True))
        ref.append(P @ vd[0] / P.sum(1, keepdims=True))
    ref = np.concatenate(ref)
    rel = lambda a: np.abs(a - ref).mean() / np.abs(ref).mean()
    print(f"\nrelative error vs fp64 attention: one level {rel(one):.4f}, two-level {rel(two):.4f}")
    assert rel(two) <= rel(one)
    assert rel(two) < 0.2


def test_second_level_exponent_is_clamped_at_minus_40(orc):
    # A tile far below the running max: k = max(floor(log2 p_t) - 10, -40) takes the clamp.
    # Every query row is (6, 0, ..., 0) (Q_hat exact, scale 1); key n has K[n, 0] = kv[n]
    # and zeros in channels 1..15, so S = 6 * kv[n] exactly (the K values -33, -42, -45
    # quantise exactly, scales 5.5, 7, 7.5).  Keys outside kv tile 2 have S = 0 (m = 0).
    # In tile 2 (keys 128..191, 64-key tiles): block A (S = -198: log2 P = -35.71) sets
    # p_t, so floor(log2 p_t) - 10 = -46 and the clamp gives k = -40; blocks B and D
    # (S = -252: log2 P = -45.45) keep a code (amax/6 * 2^40 = 0.0038 > 2^-10) and block C
    # (S = -270: log2 P = -48.69) flushes (amax/6 * 2^40 = 0.0004 < 2^-10).  Without the
    # clamp (k = -46) block C would keep a code; with a clamp at -30 blocks B and D would
    # flush.  One level flushes the whole tile.
    N, d, bc = 256, 64, 64
    kv = np.zeros(N)
    kv[128:144], kv[144:160], kv[160:176], kv[176:192] = -33.0, -42.0, -45.0, -42.0
    q = np.zeros((N, d), np.float32)
    q[:, 0] = 6.0
    k = np.zeros((N, d), np.float32)
    k[:, 0] = kv
    rng = np.random.default_rng(65)
    k[:, 16:] = rng.standard_normal((N, d - 16))
    v = rng.standard_normal((N, d)).astype(np.float32)
    bits = lambda a: gen.f32_to_bf16_bits(a)[None, None]
    qz = orc.quantize_all(bits(q), bits(k), bits(v))
    for row in (0, 200):
        two = orc.attn_trace(qz, False, bc, row, two_level=True)
        one = orc.attn_trace(qz, False, bc, row)
        t2 = two["p"][2].astype(np.float64)
        assert np.floor(np.log2(t2.max())) == -36
        ph = two["phat"][2].reshape(4, 16)
        assert np.all(ph[0] > 0) and np.all(ph[1] > 0) and np.all(ph[3] > 0), ph[:, 0]
        assert np.all(ph[2] == 0), ph[:, 0]
        assert np.all(one["phat"][2] == 0)
        # the kept blocks are within the E2M1 bound of their scale sigma_b * 2^-40
        for blk in (0, 1, 3):
            p = t2[blk * 16:(blk + 1) * 16]
            assert np.all(np.abs(ph[blk] - p) <= 0.36 * p)
