"""GPU parity of the decode / split-KV path against the oracle (or_attn_decode): the packed
query quantiser bit-exact, and the split attention + merge with m and l exact and O
within the forward path's tolerance."""
import numpy as np
import pytest
import torch

import oracle
from bit_flashattention_b200 import gen, hifa4
from tests import _layout
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

# (d, kv_tile, Hq, Hkv, nq, Nk, nsplit, smooth)
CASES = [
    (128, 256, 32, 8, 1, 2048, 4, True),      # pure decode, 4 query heads per kv head
    (128, 256, 8, 2, 32, 1024, 3, True),      # a full 128-row tile per kv head, uneven splits
    (128, 128, 4, 1, 8, 1536, 5, False),
    (64, 128, 4, 2, 3, 512, 2, False),
    (256, 64, 4, 2, 5, 384, 4, True),
    (128, 256, 4, 1, 16, 512, 1, False),      # one split: the merge is the identity
    # keys on the MMA's M dimension (head dim 128, 128-key tiles, G * nq <= 16)
    (128, 128, 32, 8, 1, 2048, 4, True),      # 4 query rows per kv head
    (128, 0, 32, 8, 1, 2048, 3, True),        # the default tile is 128 keys here
    (128, 128, 16, 2, 1, 1536, 5, False),     # 8 rows
    (128, 128, 8, 2, 4, 1024, 3, True),       # 16 rows, the last tile masked per token
    (128, 128, 4, 1, 3, 768, 2, False),       # 12 of 16 rows in use
    (128, 128, 8, 1, 1, 512, 1, True),        # one split
    (128, 0, 4, 1, 1, 128, 4, False),         # a single 128-key tile: more splits asked than tiles
    (128, 128, 16, 1, 1, 384, 2, True),       # 16 query heads per kv head, one token each
]


def _bf16(rng, shape, scale=1.0, outliers=0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    if outliers:
        ch = rng.choice(shape[-1], outliers, replace=False)
        x[..., ch] *= np.float32(8.0)
    return gen.f32_to_bf16_bits(x)


def _case(d, kv_tile, Hq, Hkv, nq, Nk, nsplit, smooth, B=2, seed=0):
    rng = np.random.default_rng(1000 + seed + d + nq)
    q = _bf16(rng, (B, Hq, nq, d))
    k = _bf16(rng, (B, Hkv, Nk, d), outliers=4)
    v = _bf16(rng, (B, Hkv, Nk, d))
    s = sinv = None
    if smooth:
        s = np.exp2(rng.uniform(-1.5, 1.5, (Hkv, d))).astype(np.float32)
        sinv = (np.float32(1.0) / s).astype(np.float32)
    return q, k, v, s, sinv


@pytest.mark.parametrize("case", CASES)
def test_decode_matches_oracle(case):
    d, kv_tile, Hq, Hkv, nq, Nk, nsplit, smooth = case
    B, G = 2, Hq // Hkv
    q, k, v, s, sinv = _case(*case, B=B)
    st = hifa4.new_status("cuda")
    dev = lambda a: None if a is None else gc.to_dev(a)
    qp = hifa4.hifa4_quantize_q_decode(gc.bf16_dev(q), Hkv, dev(s), status=st)
    kq, _ = hifa4.hifa4_quantize_qk(gc.bf16_dev(k), gc.bf16_dev(k), dev(sinv), dev(s), status=st)
    vq = hifa4.hifa4_quantize_v(gc.bf16_dev(v), status=st)
    o, m, l = hifa4.hifa4_attn_decode(qp, kq, vq, Hq, nq, kv_tile=kv_tile, nsplit=nsplit, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK

    qc, qs = oracle.quantize_rows(oracle.pack_decode_q(q, Hkv), Hkv, s)
    kc, ks = oracle.quantize_rows(k, Hkv, sinv)
    vc, vs = oracle.quantize_vt(v)
    # the packed query and the 4-bit K and V^T cache are bit-exact, codes and scales
    assert np.array_equal(qp.codes.cpu().numpy().reshape(qc.shape), qc)
    assert np.array_equal(_layout.rows_scales_to_plain(qp.scales.cpu().numpy(), B, Hkv, 128, d), qs)
    assert np.array_equal(kq.codes.cpu().numpy().reshape(kc.shape), kc)
    assert np.array_equal(_layout.rows_scales_to_plain(kq.scales.cpu().numpy(), B, Hkv, Nk, d), ks)
    assert np.array_equal(vq.codes.cpu().numpy().reshape(vc.shape), vc)
    assert np.array_equal(_layout.vt_scales_to_plain(vq.scales.cpu().numpy(), B, Hkv, Nk, d), vs)

    bc = kv_tile if kv_tile else 128
    ref = oracle.attn_decode(qc, qs, kc, ks, vc, vs, G=G, nq=nq, bc=bc, nsplit=nsplit)
    mg = m.float().cpu().numpy()
    lg = l.float().cpu().numpy()
    assert np.array_equal(mg, ref["m"])
    assert np.array_equal(lg, ref["l"])          # fp16(L), L the fp32 merge of exact fp16 partials
    og = o.view(torch.int16).cpu().numpy().view(np.uint16)
    a = gen.bf16_bits_to_f32(og).astype(np.float64)
    b = gen.bf16_bits_to_f32(ref["o_bf16"]).astype(np.float64)
    diff = np.abs(a - b)
    assert np.all(np.isfinite(a))
    assert diff.max() <= gc.O_MAX_ABS, diff.max()
    assert diff.mean() / max(np.abs(b).mean(), 1e-30) <= gc.O_MEAN_REL


def _dequant_rows(codes, scales):
    """Plain-layout 4-bit rows [.., n/2] codes, [.., n/16] scales -> float64 values."""
    import ml_dtypes
    lut = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)
    sc = scales.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return lut[nib] * np.repeat(sc, 16, axis=-1)


@pytest.mark.parametrize("kv_tile", [256, 128])
def test_decode_error_does_not_grow_with_splits(kv_tile):
    # different split counts quantise P_hat against different maxima: each count is a valid
    # evaluation, and its error against fp64 attention on the same dequantised operands stays
    # at the single-split level; the automatic count must also run (128-key tiles: the
    # kernel with keys on the MMA's M dimension)
    case = (128, kv_tile, 8, 2, 4, 4096, 1, False)
    d, kv_tile, Hq, Hkv, nq, Nk, _, _ = case
    B, G = 2, Hq // Hkv
    q, k, v, _, _ = _case(*case)
    st = hifa4.new_status("cuda")
    qp = hifa4.hifa4_quantize_q_decode(gc.bf16_dev(q), Hkv, status=st)
    kq, _ = hifa4.hifa4_quantize_qk(gc.bf16_dev(k), gc.bf16_dev(k), status=st)
    vq = hifa4.hifa4_quantize_v(gc.bf16_dev(v), status=st)
    outs = {ns: hifa4.hifa4_attn_decode(qp, kq, vq, Hq, nq, kv_tile=kv_tile, nsplit=ns, status=st)[0].float().cpu()
            .numpy() for ns in (1, 2, 7, 0)}
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    qc, qs = oracle.quantize_rows(oracle.pack_decode_q(q, Hkv), Hkv)
    kc, ks = oracle.quantize_rows(k, Hkv)
    vc, vs = oracle.quantize_vt(v)
    vdq = _dequant_rows(vc, vs)                                  # [B, Hkv, d, Nk]
    c = 1.4426950408889634 / np.sqrt(d)
    exact = np.zeros((B, Hq, nq, d))
    for b in range(B):
        for g in range(Hkv):
            S = oracle.qk_scores(qc[b, g, : G * nq], qs[b, g, : G * nq], kc[b, g], ks[b, g]).astype(np.float64)
            for r in range(G * nq):
                pos = Nk - nq + r % nq
                z = S[r, : pos + 1] * c
                p = np.exp2(z - z.max())
                exact[b, g * G + r // nq, r % nq] = vdq[b, g, :, : pos + 1] @ p / p.sum()
    err = {ns: np.abs(o - exact).mean() / np.abs(exact).mean() for ns, o in outs.items()}
    assert err[1] < 0.15, err
    for ns in (2, 7, 0):
        assert err[ns] <= 1.5 * err[1] + 0.01, err


def test_decode_rejects_bad_shapes():
    st = hifa4.new_status("cuda")
    q = torch.zeros(1, 8, 33, 128, dtype=torch.bfloat16, device="cuda")     # G * nq = 132 > 128
    with pytest.raises(hifa4.Hifa4Error):
        hifa4.hifa4_quantize_q_decode(q, 2, status=st)


@pytest.mark.parametrize("d,kv_tile,nsplit", [(128, 0, 1), (128, 0, 2), (128, 256, 1), (64, 64, 3)])
def test_decode_worked_example_from_the_golden_fixture(d, kv_tile, nsplit):
    # the hand-derived decode case of tests/golden/worked_examples.txt: Q = 0 against the
    # fixture's V over 256 keys gives m = 0, l = 264 and O = 0.09375 * 2^-(c % 4) at any
    # split count (kv_tile 0 at d = 128: the kernel with the keys on the MMA's M dimension)
    from tests import _golden
    sec = _golden.load()["decode_q_zero"]
    _, k, v, _ = _golden.attn_inputs(256, d)
    st = hifa4.new_status("cuda")
    q = torch.zeros(1, 1, 1, d, dtype=torch.bfloat16, device="cuda")
    qp = hifa4.hifa4_quantize_q_decode(q, 1, status=st)
    kq, _ = hifa4.hifa4_quantize_qk(gc.bf16_dev(k), gc.bf16_dev(k), status=st)
    vq = hifa4.hifa4_quantize_v(gc.bf16_dev(v), status=st)
    o, m, l = hifa4.hifa4_attn_decode(qp, kq, vq, 1, 1, kv_tile=kv_tile, nsplit=nsplit, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    u16 = lambda t: t.reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)
    assert u16(m)[0] == _golden.num(sec["m_fp16"][0])
    assert u16(l)[0] == _golden.num(sec["l_fp16"][0])
    want = np.array([_golden.num(b) for b in sec["o_bf16_by_c_mod_4"]], np.uint16)[np.arange(d) % 4]
    assert np.array_equal(u16(o), want)
