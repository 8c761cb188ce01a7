"""Pins of the oracle's block quantiser, Smooth-QK calibration/application and the
4-bit dot product (S) against library routines, invariants and closed forms."""
import ml_dtypes
import numpy as np

from bit_flashattention_b200 import configs, gen


def _dequant(codes, scales):
    """Dequantise with ml_dtypes (library decode of E2M1 and E4M3)."""
    lo = (codes & 0xF).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    hi = (codes >> 4).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    v = np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)
    s = scales.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    return v * np.repeat(s, 16, axis=-1)


def test_block_amax_element_gets_top_code(orc):
    # For a block whose scale is an E4M3 normal, amax/scale lies in 6*[1-2^-4, 1+2^-4],
    # which E2M1 rounds to 6 (code 7): the largest element always uses the top code.
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((20000, 16)) * 10.0 ** rng.uniform(-1, 2, (20000, 1))).astype(np.float32)
    codes, scales = orc.quant_blocks(x.ravel())
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(20000, 16)
    top = np.abs(x).argmax(1)
    assert np.all((nib[np.arange(20000), top] & 7) == 7)
    assert np.all(scales >= 0x08)                    # normal E4M3 scales for these magnitudes


def test_block_scale_equivariance(orc):
    # Multiplying a block by 2^k (scale stays an E4M3 normal) leaves the codes unchanged
    # and moves the scale's exponent by k: the scale really is amax/6 and codes use 1/scale.
    rng = np.random.default_rng(5)
    x = rng.uniform(-3, 3, (5000, 16)).astype(np.float32)
    c0, s0 = orc.quant_blocks(x.ravel())
    for k in (-3, 1, 4):
        ck, sk = orc.quant_blocks((x * np.float32(2.0 ** k)).ravel())
        assert np.array_equal(c0, ck)
        assert np.array_equal(sk.astype(int) - s0.astype(int), np.full(s0.shape, 8 * k))


def test_block_dequant_error_bound(orc):
    # |x - dequant(x)| <= half the E2M1 gap at that magnitude times the scale (no saturation
    # beyond the top code for amax, whose excess is bounded by the scale rounding).
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(160000)).astype(np.float32)
    codes, scales = orc.quant_blocks(x)
    xd = _dequant(codes[None], scales[None])[0]
    sig = np.repeat(scales.view(ml_dtypes.float8_e4m3fn).astype(np.float32), 16)
    assert np.all(np.abs(x - xd) <= 1.0 * sig * 1.07 + 1e-30)
    # relative Frobenius error of NVFP4 on Gaussian data is ~10%
    assert np.linalg.norm(x - xd) / np.linalg.norm(x) < 0.15


def test_quantize_rows_applies_group_channel_scale(orc):
    # Power-of-two scales make x*s exact, so smoothing inside the quantiser must equal
    # quantising the numpy product: pins the (kv group, channel) indexing of s.
    B, H, Hkv, N, d = 2, 4, 2, 32, 64
    rng = np.random.default_rng(7)
    x = gen.f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32))
    s = np.float32(2.0) ** rng.integers(-3, 4, (Hkv, d)).astype(np.float32)
    c1, s1 = orc.quantize_rows(x, Hkv, s)
    xs = gen.bf16_bits_to_f32(x) * np.repeat(s, H // Hkv, axis=0)[None, :, None, :]
    c2, s2 = orc.quant_blocks(xs.ravel())
    assert np.array_equal(c1.ravel(), c2) and np.array_equal(s1.ravel(), s2)


def test_quantize_vt_is_blocks_along_tokens(orc):
    B, Hkv, N, d = 1, 2, 64, 32
    rng = np.random.default_rng(8)
    v = gen.f32_to_bf16_bits(rng.standard_normal((B, Hkv, N, d)).astype(np.float32))
    c1, s1 = orc.quantize_vt(v)
    vt = np.ascontiguousarray(np.swapaxes(gen.bf16_bits_to_f32(v), 2, 3))
    c2, s2 = orc.quant_blocks(vt.ravel())
    assert np.array_equal(c1.ravel(), c2) and np.array_equal(s1.ravel(), s2)


def test_calibrate_properties(orc):
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=8, Hkv=2, N=256)
    q, k, _ = gen.inputs(w, calib=True)
    s0, si0 = orc.calibrate(q, k, 0.0)
    assert np.all(s0 == 1.0) and np.all(si0 == 1.0)            # alpha = 0 disables smoothing
    s, si = orc.calibrate(q, k, 0.5)
    assert np.array_equal(si, (np.float32(1.0) / s).astype(np.float32))
    # balanced point: after smoothing, per-(group, channel) amax of Q*s and K/s agree
    qf, kf = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k)
    grp = w.Hq // w.Hkv
    aq = np.abs(qf).reshape(w.B, w.Hkv, grp, w.N, w.d).max(axis=(0, 2, 3))
    ak = np.abs(kf).max(axis=(0, 2))
    assert np.allclose(aq * s, ak / s, rtol=1e-6)
    # scaling K by 4 (exact in bf16) scales s by 4^0.5 = 2 exactly
    k4 = gen.f32_to_bf16_bits(kf * 4)
    s4, _ = orc.calibrate(q, k4, 0.5)
    assert np.array_equal(s4, s * 2)


def test_s_dot_models_on_exact_cases(orc):
    # With unit scales and small codes every partial sum is exact, so all three
    # accumulation models must equal numpy's matmul of the dequantised operands.
    rng = np.random.default_rng(9)
    for d in (64, 128, 256):
        qc = rng.integers(0, 256, (16, d // 2), dtype=np.uint8)
        kc = rng.integers(0, 256, (24, d // 2), dtype=np.uint8)
        qs = np.full((16, d // 16), 0x38, np.uint8)
        ks = np.full((24, d // 16), 0x38, np.uint8)
        ref = (_dequant(qc, qs).astype(np.float64) @ _dequant(kc, ks).astype(np.float64).T).astype(np.float32)
        for model in (0, 1, 2, 3):
            assert np.array_equal(orc.qk_scores(qc, qs, kc, ks, model), ref)


def test_s_dot_exact_model_is_rounded_exact_dot(orc):
    # Scales within a 2^6 range keep the fp64 dot of dequantised values exact, so the
    # "exact then one rounding" model must equal RN(numpy fp64 matmul).
    rng = np.random.default_rng(10)
    d = 128
    qc = rng.integers(0, 256, (32, d // 2), dtype=np.uint8)
    kc = rng.integers(0, 256, (40, d // 2), dtype=np.uint8)
    qs = rng.integers(0x30, 0x50, (32, d // 16), dtype=np.uint8)
    ks = rng.integers(0x30, 0x50, (40, d // 16), dtype=np.uint8)
    ref = (_dequant(qc, qs).astype(np.float64) @ _dequant(kc, ks).astype(np.float64).T).astype(np.float32)
    assert np.array_equal(orc.qk_scores(qc, qs, kc, ks, 2), ref)
    for model in (0, 1):
        got = orc.qk_scores(qc, qs, kc, ks, model).astype(np.float64)
        assert np.all(np.abs(got - ref) <= 2 * np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64))


def _rz_f32(num: int, den_log2: int) -> float:
    """num * 2^-den_log2 rounded toward zero to fp32, with Python integers."""
    a = abs(num)
    n = a.bit_length()
    if n > 24:
        a = (a >> (n - 24)) << (n - 24)
    return float(np.float32((-a if num < 0 else a) * 2.0 ** -den_log2))


def test_s_dot_rz_model_against_integer_arithmetic(orc):
    # Model 3 (per 64-chunk: acc = RZ(acc + exact chunk)) recomputed with Python big
    # integers from the format definitions, on wide-range scales where rounding matters.
    rng = np.random.default_rng(12)
    E2 = [0, 1, 2, 3, 4, 6, 8, 12]
    tw = lambda c: -E2[c & 7] if c & 8 else E2[c & 7]
    sc = lambda b: (b & 7) if (b >> 3) == 0 else (8 + (b & 7)) << ((b >> 3) - 1)
    for d in (64, 128, 256):
        qc = rng.integers(0, 256, (8, d // 2), dtype=np.uint8)
        kc = rng.integers(0, 256, (8, d // 2), dtype=np.uint8)
        qs = rng.integers(1, 0x7F, (8, d // 16), dtype=np.uint8)
        ks = rng.integers(1, 0x7F, (8, d // 16), dtype=np.uint8)
        got = orc.qk_scores(qc, qs, kc, ks, 3)
        for i in range(8):
            for k in range(8):
                qn = [(int(qc[i, e // 2]) >> (4 * (e & 1))) & 15 for e in range(d)]
                kn = [(int(kc[k, e // 2]) >> (4 * (e & 1))) & 15 for e in range(d)]
                acc = 0.0
                for ch in range(d // 64):
                    t = 0
                    for b in range(4 * ch, 4 * ch + 4):
                        isum = sum(tw(qn[16 * b + e]) * tw(kn[16 * b + e]) for e in range(16))
                        t += isum * sc(int(qs[i, b])) * sc(int(ks[k, b]))
                    acc = _rz_f32(int(round(acc * 2 ** 20)) + t, 20)
                assert got[i, k] == np.float32(acc)


def test_smooth_qk_leaves_qkt_unchanged_in_exact_arithmetic(orc):
    # (Q*s)(K/s)^T = QK^T.  Exactly representable case: s constant over each 16-channel
    # block and a power of two, so Q*s and K/s are exact, each block's codes are unchanged
    # and its E4M3 scale moves by the same power of two in opposite directions (scales stay
    # normal here); the exact 4-bit dot products, and so the whole quantised attention,
    # must then be bit-identical with and without Smooth-QK.
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=4, Hkv=2, N=256, d=128, bc=64)
    q, k, v = gen.inputs(w)
    rng = np.random.default_rng(10)
    e = rng.integers(-2, 3, (w.Hkv, w.d // 16))
    s = np.repeat(np.float32(2.0) ** e.astype(np.float32), 16, axis=1)
    sinv = (np.float32(1.0) / s).astype(np.float32)
    plain = orc.quantize_all(q, k, v)
    smooth = orc.quantize_all(q, k, v, s, sinv)
    assert np.array_equal(plain.qc, smooth.qc) and np.array_equal(plain.kc, smooth.kc)
    g = np.repeat(np.arange(w.Hkv), w.Hq // w.Hkv)
    assert np.array_equal(smooth.qs.astype(int) - plain.qs.astype(int), np.broadcast_to(8 * e[g][None, :, None, :],
                                                                                          plain.qs.shape))
    assert np.array_equal(smooth.ks.astype(int) - plain.ks.astype(int), np.broadcast_to(-8 * e[None, :, None, :],
                                                                                          plain.ks.shape))
    for h in range(w.Hq):
        S0 = orc.qk_scores(plain.qc[0, h], plain.qs[0, h], plain.kc[0, g[h]], plain.ks[0, g[h]], 2)
        S1 = orc.qk_scores(smooth.qc[0, h], smooth.qs[0, h], smooth.kc[0, g[h]], smooth.ks[0, g[h]], 2)
        assert np.array_equal(S0, S1)
    a, b = orc.attn_fwd(plain, True, w.bc), orc.attn_fwd(smooth, True, w.bc)
    assert all(np.array_equal(a[x], b[x]) for x in ("o_bf16", "m", "l"))
    # and with the calibrated (not power-of-two) s, fp64 (Q*s)(K*s_inv)^T stays within the
    # rounding of s_inv = RN(1/s) of QK^T
    qc, kc, _ = gen.inputs(w, calib=True)
    sc, sci = orc.calibrate(qc, kc, 0.5)
    qf = gen.bf16_bits_to_f32(q).astype(np.float64)[0]
    kf = gen.bf16_bits_to_f32(k).astype(np.float64)[0]
    for h in range(w.Hq):
        ref = qf[h] @ kf[g[h]].T
        got = (qf[h] * sc[g[h]]) @ (kf[g[h]] * sci[g[h]]).T
        bound = np.abs(qf[h]) @ np.abs(kf[g[h]]).T * 2.0 ** -23
        assert np.all(np.abs(got - ref) <= bound)
