"""Pins of the oracle's decode / split-KV attention (or_attn_decode): packed query rows,
visibility of the keys up to each token's position, the split tile ranges and the fp32
merge of the per-split (m, l, O) partials."""
import numpy as np

from bit_flashattention_b200 import gen


def _bf16(rng, shape, scale=1.0):
    return gen.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _quant(orc, qdec, k, v, Hkv):
    qp = orc.pack_decode_q(qdec, Hkv)
    qc, qs = orc.quantize_rows(qp, Hkv)
    kc, ks = orc.quantize_rows(k, Hkv)
    vc, vs = orc.quantize_vt(v)
    return qc, qs, kc, ks, vc, vs


def test_single_split_equals_the_square_forward(orc):
    # token t of the decode query sits at position Nk - nq + t: with one split its output is
    # the square causal forward's row Nk - nq + t on the same quantised operands
    rng = np.random.default_rng(41)
    B, Hq, Hkv, nq, Nk, d, bc = 1, 4, 2, 8, 512, 64, 64
    G = Hq // Hkv
    qdec = _bf16(rng, (B, Hq, nq, d))
    k = _bf16(rng, (B, Hkv, Nk, d))
    v = _bf16(rng, (B, Hkv, Nk, d))
    dec = orc.attn_decode(*_quant(orc, qdec, k, v, Hkv), G=G, nq=nq, bc=bc, nsplit=1)
    qsq = np.zeros((B, Hq, Nk, d), np.uint16)
    qsq[:, :, Nk - nq:] = qdec
    qz = orc.quantize_all(qsq, k, v)
    rows = np.array([(h * Nk) + Nk - nq + t for h in range(Hq) for t in range(nq)], np.int64)
    ref = orc.attn_fwd(qz, True, bc, rows)
    assert np.array_equal(dec["m"].reshape(-1), ref["m"])
    assert np.array_equal(dec["l"].reshape(-1), ref["l"])
    # out = bf16(O * RN(1/L)) here, bf16(O / l) in the square forward: at most one bf16 ulp
    a = gen.bf16_bits_to_f32(dec["o_bf16"].reshape(-1, d)).astype(np.float64)
    b = gen.bf16_bits_to_f32(ref["o_bf16"].reshape(-1, d)).astype(np.float64)
    assert np.all(np.abs(a - b) <= np.spacing(np.abs(b).astype(np.float32)).astype(np.float64) * 2 ** 16 + 1e-30)
    assert np.mean(a == b) > 0.99


def test_first_split_partial_is_the_forward_over_its_keys(orc):
    # split 0 of 2 covers tiles [0, T); every decode token sees all of those keys, so its
    # partial equals the non-causal forward over the first T * bc keys alone
    rng = np.random.default_rng(42)
    B, Hq, Hkv, nq, Nk, d, bc = 1, 2, 1, 4, 512, 64, 128
    G = Hq // Hkv
    qdec = _bf16(rng, (B, Hq, nq, d))
    k = _bf16(rng, (B, Hkv, Nk, d))
    v = _bf16(rng, (B, Hkv, Nk, d))
    dec = orc.attn_decode(*_quant(orc, qdec, k, v, Hkv), G=G, nq=nq, bc=bc, nsplit=2)
    T = (Nk // bc + 1) // 2
    n0 = T * bc
    qsq = np.zeros((B, Hq, n0, d), np.uint16)
    qsq[:, :, :nq] = qdec
    qz = orc.quantize_all(qsq, k[:, :, :n0], v[:, :, :n0])
    rows = np.array([h * n0 + t for h in range(Hq) for t in range(nq)], np.int64)
    ref = orc.attn_fwd(qz, False, bc, rows)
    pml = dec["part_ml"].reshape(B * Hkv, 2, 128, 2)[0, 0, : G * nq]
    assert np.array_equal(pml[:, 0], ref["m"]) and np.array_equal(pml[:, 1], ref["l"])
    po = dec["part_o"].reshape(B * Hkv, 2, 128, d)[0, 0, : G * nq].astype(np.float64)
    o_ref = gen.bf16_bits_to_f32(ref["o_bf16"]).astype(np.float64)
    assert np.allclose(po / pml[:, 1:2], o_ref, rtol=2 ** -7, atol=1e-6)


def test_constant_values_survive_any_split(orc):
    # V = 1 everywhere: every P_hat row is a weighted mean of the same dequantised value
    # (1.0 -> code 6 with scale E4M3(1/6) = 0.171875 -> 1.03125), so the merged output is
    # exactly that value for any number of splits, including splits with no visible key
    rng = np.random.default_rng(43)
    B, Hq, Hkv, nq, Nk, d, bc = 2, 4, 1, 3, 384, 64, 64
    G = Hq // Hkv
    qdec = _bf16(rng, (B, Hq, nq, d), scale=2.0)
    k = _bf16(rng, (B, Hkv, Nk, d), scale=2.0)
    v = gen.f32_to_bf16_bits(np.ones((B, Hkv, Nk, d), np.float32))
    ops = _quant(orc, qdec, k, v, Hkv)
    for nsplit in (1, 2, 4, 7):
        dec = orc.attn_decode(*ops, G=G, nq=nq, bc=bc, nsplit=nsplit)
        out = gen.bf16_bits_to_f32(dec["o_bf16"])
        assert np.all(out == np.float32(1.03125)), nsplit
        assert np.all(dec["l"] > 0)


def test_merge_weights_follow_the_softmax_mass(orc):
    # V = 1 on the keys of split 0 and 0 on those of split 1: the merged output is the
    # dequantised 1 (1.03125) times the share of the softmax mass on split 0, which an fp64
    # softmax over the exact 4-bit scores gives to within the P_hat quantisation error.
    # Split 1's keys are scaled down, so the two splits' maxima differ by several units and a
    # wrong merge weight (e.g. E(m - m_s)) moves the share far outside the bound.
    rng = np.random.default_rng(44)
    B, Hq, Hkv, nq, Nk, d, bc = 1, 2, 1, 2, 256, 64, 64
    G = Hq // Hkv
    qdec = _bf16(rng, (B, Hq, nq, d), scale=1.5)
    kf = rng.standard_normal((B, Hkv, Nk, d)).astype(np.float32) * 1.5
    kf[:, :, 128:] *= 0.25
    k = gen.f32_to_bf16_bits(kf)
    vf = np.zeros((B, Hkv, Nk, d), np.float32)
    vf[:, :, :128] = 1.0
    v = gen.f32_to_bf16_bits(vf)
    qc, qs, kc, ks, vc, vs = _quant(orc, qdec, k, v, Hkv)
    dec = orc.attn_decode(qc, qs, kc, ks, vc, vs, G=G, nq=nq, bc=bc, nsplit=2)
    out = gen.bf16_bits_to_f32(dec["o_bf16"]).astype(np.float64)
    c = 1.4426950408889634 / np.sqrt(d)
    shares = []
    for h in range(Hq):
        for t in range(nq):
            r = h * nq + t
            S = orc.qk_scores(qc[0, 0, r:r + 1], qs[0, 0, r:r + 1], kc[0, 0], ks[0, 0]).astype(np.float64)[0]
            pos = Nk - nq + t
            z = S[: pos + 1] * c
            p = np.exp2(z - z.max())
            share = p[:128].sum() / p.sum()
            shares.append(share)
            got = out[0, h, t] / 1.03125
            assert np.all(np.abs(got - share) <= 0.04), (h, t, share, got[:4])
    assert 0.3 < min(shares) and max(shares) < 0.995
