"""The oracle against the hand-derived worked examples in tests/golden/worked_examples.txt:
the E2M1 and E4M3 element types, the 16-element block quantiser (exact, flushed and
clipped blocks), the Smooth-QK calibration, and two attention cases whose every step has
a closed form (Q = 0 over a V that quantises exactly, and the first causal row).  The
expected values are the fixture's; the inputs are built here from the recipes the fixture
states."""
import numpy as np
import pytest

from bit_flashattention_b200 import gen
from tests._golden import attn_inputs as _attn_inputs, load, num as _num

G = load()


def test_fixture_has_every_section():
    assert set(G) == {"e2m1_decode", "e2m1_encode", "e4m3_decode", "e4m3_encode", "block_exact", "block_flushed",
                      "block_clipped", "calibration", "attn_q_zero", "attn_causal_row0", "decode_q_zero", "attn_select",
                      "attn_bf16_tie"}


def test_e2m1_decode(orc):
    for code, (val,) in G["e2m1_decode"].items():
        got = orc.e2m1_value(int(code))
        assert got == float(val) and np.signbit(got) == val.startswith("-"), (code, got, val)


def test_e2m1_encode(orc):
    xs = np.array([float(x) for x in G["e2m1_encode"]], np.float32)
    want = np.array([int(v[0]) for v in G["e2m1_encode"].values()], np.uint8)
    assert np.array_equal(orc.e2m1_encode(xs), want), (xs, orc.e2m1_encode(xs), want)


def test_e4m3_decode_and_encode(orc):
    for code, (val,) in G["e4m3_decode"].items():
        assert orc.e4m3_value(int(code, 16)) == float(val), code
    xs = np.array([float(x) for x in G["e4m3_encode"]], np.float32)
    want = np.array([_num(v[0]) for v in G["e4m3_encode"].values()], np.uint8)
    assert np.array_equal(orc.e4m3_encode(xs), want), (xs, orc.e4m3_encode(xs), want)
    # the fixture's fp32 values are the roundings it names
    assert np.float32(1.0) / np.float32(6.0) == np.float32(0.1666666716337204)
    assert np.float32(1000.0) * (np.float32(1.0) / np.float32(6.0)) == np.float32(166.66667175292969)


@pytest.mark.parametrize("name,key,factor", [("block_exact", "x_times_16", 1 / 16),
                                             ("block_flushed", "x_times_8192", 1 / 8192),
                                             ("block_clipped", "x", 1.0)])
def test_block_quantiser(orc, name, key, factor):
    sec = G[name]
    x = np.array([float(v) for v in sec[key]], np.float64) * factor
    codes, scales = orc.quant_blocks(x.astype(np.float32))
    assert scales.tolist() == [_num(sec["scale"][0])]
    assert codes.tolist() == [_num(b) for b in sec["bytes"]]


def test_calibration(orc):
    sec = G["calibration"]
    B, Hq, Hkv, N, d = 1, 2, 1, 16, 64
    q = np.zeros((B, Hq, N, d), np.float32)
    k = np.zeros((B, Hkv, N, d), np.float32)
    want = {}
    for c in range(d):
        aq, ak, s, si = (float(v) for v in sec.get(f"channel_{c}", sec["other_channels"]))
        # the amax sits on a different token (and, for Q, query head) per channel; the
        # rest of the column is smaller and of mixed sign
        q[0, c % 2, (3 * c) % N, c] = aq
        q[0, (c + 1) % 2, (5 * c + 1) % N, c] = -aq / 2
        k[0, 0, (7 * c + 2) % N, c] = -ak
        k[0, 0, (7 * c + 3) % N, c] = ak / 4
        want[c] = (s, si)
    s, sinv = orc.calibrate(gen.f32_to_bf16_bits(q), gen.f32_to_bf16_bits(k), 0.5)
    for c in range(d):
        assert (s[0, c], sinv[0, c]) == want[c], (c, s[0, c], sinv[0, c], want[c])


@pytest.mark.parametrize("bc", [16, 64, 256])
def test_attention_with_zero_queries(orc, bc):
    sec = G["attn_q_zero"]
    q, k, v, _ = _attn_inputs()
    qz = orc.quantize_all(q, k, v)
    assert np.array_equal(qz.qc, np.zeros_like(qz.qc)) and np.array_equal(qz.qs, np.zeros_like(qz.qs))
    ref = orc.attn_fwd(qz, False, bc)
    assert np.all(ref["m16"] == _num(sec["m_fp16"][0]))
    assert np.all(ref["l16"] == _num(sec["l_fp16"][0]))
    want = np.array([_num(b) for b in sec["o_bf16_by_c_mod_4"]], np.uint16)[np.arange(64) % 4]
    assert np.all(ref["o_bf16"] == want[None, :]), ref["o_bf16"][0]
    # every key's P is 1 and its dequantised P_hat is the fixture's code times its scale
    phat = float(G["e2m1_decode"][sec["phat_code"][0]][0]) * float(G["e4m3_decode"][sec["phat_scale"][0]][0])
    assert phat == 1.03125
    t = orc.attn_trace(qz, False, bc, 77)
    assert np.all(t["p"] == 1.0) and np.all(t["phat"] == phat), t["phat"][:1]


def test_first_causal_row(orc):
    sec = G["attn_causal_row0"]
    q, k, v, vf = _attn_inputs()
    ref = orc.attn_fwd(orc.quantize_all(q, k, v), True, 64, [0])
    assert ref["m16"][0] == _num(sec["m_fp16"][0]) and ref["l16"][0] == _num(sec["l_fp16"][0])
    got = gen.bf16_bits_to_f32(ref["o_bf16"][0])
    assert got[:16].tolist() == [float(x) for x in sec["o_first_16"]]
    assert np.array_equal(got, vf[0].astype(np.float32))
    t = orc.attn_trace(orc.quantize_all(q, k, v), True, 64, 0)
    assert t["phat"].shape == (1, 64) and t["phat"][0, 0] == 1.03125 and np.all(t["phat"][0, 1:] == 0)


@pytest.mark.parametrize("d,bc,nsplit", [(64, 64, 1), (64, 64, 3), (128, 128, 2), (128, 256, 1), (128, 16, 16)])
def test_decode_with_zero_query(orc, d, bc, nsplit):
    sec = G["decode_q_zero"]
    _, k, v, _ = _attn_inputs(256, d)
    q = np.zeros((1, 1, 1, d), np.uint16)
    qc, qs = orc.quantize_rows(orc.pack_decode_q(q, 1), 1)
    kc, ks = orc.quantize_rows(k, 1)
    vc, vs = orc.quantize_vt(v)
    ref = orc.attn_decode(qc, qs, kc, ks, vc, vs, G=1, nq=1, bc=bc, nsplit=nsplit)
    assert ref["m"].astype(np.float16).view(np.uint16)[0, 0, 0] == _num(sec["m_fp16"][0])
    assert ref["l"].astype(np.float16).view(np.uint16)[0, 0, 0] == _num(sec["l_fp16"][0])
    want = np.array([_num(b) for b in sec["o_bf16_by_c_mod_4"]], np.uint16)[np.arange(d) % 4]
    assert np.array_equal(ref["o_bf16"][0, 0, 0], want)


@pytest.mark.parametrize("bc", [16, 64, 256])
def test_attention_over_selected_keys(orc, bc):
    from tests import _golden
    sec = G["attn_select"]
    q, k, v, _ = _golden.select_inputs()
    qz = orc.quantize_all(q, k, v)
    assert qz.qs[0, 0, 0, 0] == 0x38 and qz.qc[0, 0, 0, 0] == 7
    assert np.all(qz.ks[0, 0, 1::4, 0] == 0x38) and np.all(qz.ks[0, 0, 0::4, 0] == 0)
    ref = orc.attn_fwd(qz, False, bc)
    assert np.all(ref["m16"] == _num(sec["m_fp16"][0]))
    assert np.all(ref["l16"] == _num(sec["l_fp16"][0]))
    want = np.array([_num(b) for b in sec["o_bf16_by_c_mod_4"]], np.uint16)[np.arange(64) % 4]
    assert np.all(ref["o_bf16"] == want[None, :]), ref["o_bf16"][0][:4]
    t = orc.attn_trace(qz, False, bc, 5)
    sel = (np.arange(256) % 4 == 0).reshape(-1, bc)
    assert np.all(t["phat"][sel] == 1.03125) and np.all(t["phat"][~sel] == 0)
    assert np.all(np.abs(t["p"][~sel] - 2.0 ** (-36 * np.float32(np.log2(np.e) / 8))) < 1e-3)


@pytest.mark.parametrize("bc", [64, 256])
def test_output_rounds_a_tie_to_even(orc, bc):
    from tests import _golden
    sec = G["attn_bf16_tie"]
    q, k, v = _golden.tie_inputs()
    qz = orc.quantize_all(q, k, v)
    assert np.all(qz.vs == 0x28)
    ref = orc.attn_fwd(qz, False, bc, want_f64=True)
    assert np.all(ref["m16"] == _num(sec["m_fp16"][0])) and np.all(ref["l16"] == _num(sec["l_fp16"][0]))
    assert np.all(ref["o_f64"] == 1.0 + 2.0 ** -8)          # O / l before the bf16 rounding
    assert np.all(ref["o_bf16"] == _num(sec["o_bf16"][0]))
