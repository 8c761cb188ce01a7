"""GPU parity of the fused 4-bit attention forward against the oracle, through the C ABI:
FP16 m and l exact per row, O within max-abs 1e-2 and mean-relative 1e-3, on seeded
synthetic inputs of every workload family (reduced sizes compared on every row; full
sizes on sampled rows), plus the bounded-wait timeout path."""
import numpy as np
import pytest
import torch

from bit_flashattention_b200 import configs, gen, hifa4, hifa4_testhooks as th
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

REDUCED = [
    ("tiny", {}),
    ("tiny", dict(causal=True)),
    ("qwen3-8b-4k", dict(Hq=4, Hkv=2, N=512)),
    ("qwen3-8b-4k", dict(Hq=4, Hkv=2, N=512, bc=128)),
    ("qwen3-8b-4k", dict(Hq=4, Hkv=2, N=384, bc=128, causal=False)),
    ("qwen3-8b-4k", dict(Hq=2, Hkv=1, N=768, causal=False)),
    ("qwen3-8b-4k", dict(Hq=2, Hkv=1, N=256, bc=64)),
    ("gemma2-9b-8k", dict(Hq=4, Hkv=2, N=512)),
    ("gemma2-9b-8k", dict(Hq=2, Hkv=1, N=256, causal=False)),
    ("llama3.1-8b-b4-16k", dict(B=2, Hq=4, Hkv=1, N=512)),
    ("phi-32k", dict(Hq=3, Hkv=1, N=1024)),
    ("tiny", dict(d=64, bc=128, N=512, causal=True)),
]


@pytest.mark.parametrize("name,kw", REDUCED)
def test_parity_reduced_all_rows(name, kw):
    w = configs.scaled(configs.get(name), **kw)
    gc.assert_parity(gc.run_parity(w))


@pytest.mark.parametrize("name", configs.ORDER)
def test_parity_full_size_sampled_rows(name):
    # every workload at its full size; rows: the first and last 128-row query tile and 4
    # seeded random rows of every (batch, head)
    w = configs.get(name)
    rows = gen.sample_rows(w, per_head=4) if w.N > 256 else None
    gc.assert_parity(gc.run_parity(w, rows, check_quant=False))


def test_parity_full_size_128_key_tiles_sampled_rows():
    # the full Qwen3-8B-shaped 4k call at 128-key tiles (32 score columns per softmax warp)
    w = configs.scaled(configs.get("qwen3-8b-4k"), bc=128)
    gc.assert_parity(gc.run_parity(w, gen.sample_rows(w, per_head=4), check_quant=False))


EDGE = [
    ("qwen3-8b-4k", dict(Hq=2, Hkv=1, N=128, bc=128)),                 # one query tile, one kv tile
    ("qwen3-8b-4k", dict(Hq=2, Hkv=1, N=128, bc=128, causal=False)),
    ("qwen3-8b-4k", dict(Hq=2, Hkv=1, N=256)),                         # 256-key tile, q-tile 0 half masked
    ("qwen3-8b-4k", dict(Hq=4, Hkv=4, N=512)),                         # no GQA
    ("llama3.1-8b-b4-16k", dict(B=3, Hq=2, Hkv=2, N=512, causal=False)),
    ("gemma2-9b-8k", dict(B=2, Hq=2, Hkv=1, N=128)),                   # d = 256, two 64-key tiles
    ("qwen3-8b-4k", dict(B=2, Hq=4, Hkv=2, N=768, bc=64)),             # d = 128, 64-key tiles: two CTAs per SM
]


@pytest.mark.parametrize("name,kw", EDGE)
def test_parity_edge_shapes(name, kw):
    w = configs.scaled(configs.get(name), **kw)
    gc.assert_parity(gc.run_parity(w))


def _parity_custom(w, q, k, v, s=None, sinv=None, v_dev=None):
    import oracle
    qq, kq, vq, vt = gc.gpu_quantize(w, q, k, v, s, sinv)
    qz = oracle.quantize_all(q, k, v, s, sinv)
    res = gc.oracle_from_gpu_layout_check(w, qq, kq, vq, qz)
    assert all(res.values()), res
    o, m, l, code = gc.gpu_attention(w, qq, kq, vt if v_dev is None else v_dev)
    assert code == hifa4.OK, hifa4.status_string(code)
    rows = np.arange(w.B * w.Hq * w.N, dtype=np.int64)
    ref = oracle.attn_fwd(qz, w.causal, w.bc, rows)
    return gc.compare_outputs(w, rows, o, m, l, ref), o


def test_zero_values_give_zero_output():
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=2, Hkv=1, N=512)
    q, k, v = gen.inputs(w)
    stats, o = _parity_custom(w, q, k, np.zeros_like(v))
    gc.assert_parity(stats)
    assert float(o.float().abs().max()) == 0.0


def test_large_and_widely_spread_scores():
    # Q scaled by 8 and one K channel by 30: scores reach a few thousand (scaled max ~500,
    # inside the FP16 range of m) and span far more than 127 in log2 units, so the exponent
    # argument saturates and many blocks get the zero scale.
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=2, Hkv=1, N=512)
    q, k, v = gen.inputs(w)
    qf = gen.bf16_bits_to_f32(q) * 8.0
    kf = gen.bf16_bits_to_f32(k)
    kf[..., 3] *= 30.0
    stats, _ = _parity_custom(w, gen.f32_to_bf16_bits(qf), gen.f32_to_bf16_bits(kf), v)
    gc.assert_parity(stats)


def test_strided_value_input():
    # V as a permuted view of a [B, N, H, d] buffer goes straight into hifa4_attn_fwd
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=4, Hkv=2, N=512)
    q, k, v = gen.inputs(w)
    v_view = gc.bf16_dev(np.ascontiguousarray(v.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
    assert not v_view.is_contiguous()
    stats, _ = _parity_custom(w, q, k, v, v_dev=v_view)
    gc.assert_parity(stats)


@pytest.mark.parametrize("bc", [256, 128])
def test_timeout_is_reported_and_context_survives(bc):
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=2, Hkv=1, N=512, bc=bc)
    q, k, v = gen.inputs(w)
    qq, kq, vq, vt = gc.gpu_quantize(w, q, k, v, None, None)
    # the injection is an argument of the test library's entry point, with that library's
    # own (shortened) wait limit: the product library's calls are untouched
    th.set_wait_limit_ns(200_000_000)
    try:
        st = hifa4.new_status("cuda")
        th.attn_fwd_inject(qq, kq, vq, causal=w.causal, kv_tile=w.bc, inject=1, status=st)
        code = hifa4.hifa4_read_status(st)
    finally:
        th.set_wait_limit_ns(2_000_000_000)
    assert code == hifa4.ERR_TIMEOUT
    # without the injection the same test entry point is the plain forward
    st = hifa4.new_status("cuda")
    o1, m1, l1 = th.attn_fwd_inject(qq, kq, vq, causal=w.causal, kv_tile=w.bc, inject=0, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    o2, m2, l2, code2 = gc.gpu_attention(w, qq, kq, vt)
    assert code2 == hifa4.OK
    assert torch.equal(o1, o2) and torch.equal(m1, m2) and torch.equal(l1, l2)
    # the context is still usable and the next call is correct
    gc.assert_parity(gc.run_parity(w))


@pytest.mark.parametrize("zero_q", [True, False])
def test_maximum_length(zero_q):
    # the longest supported sequence, N = 63488 (N * 1.03 < 65504 keeps the FP16 l finite),
    # causal with 256-key tiles, on sampled rows including the last.  With Q = 0 every
    # score is 0: P_hat = 1.03125 for every visible key, and the last row's FP16 l, summed
    # tile by tile with one FP16 rounding each, ends just under the FP16 maximum
    import oracle
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=1, Hkv=1, N=63488)
    q, k, v = gen.inputs(w)
    if zero_q:
        q = np.zeros_like(q)
    qq, kq, vq, vt = gc.gpu_quantize(w, q, k, v, None, None)
    o, m, l, code = gc.gpu_attention(w, qq, kq, vt)
    assert code == hifa4.OK, hifa4.status_string(code)
    qz = oracle.quantize_all(q, k, v)
    rows = np.array([0, 1, 255, 256, 31000, w.N - 257, w.N - 2, w.N - 1], np.int64)
    ref = oracle.attn_fwd(qz, w.causal, w.bc, rows)
    gc.assert_parity(gc.compare_outputs(w, rows, o, m, l, ref))
    lg = l.reshape(-1).float()
    assert bool(torch.isfinite(lg).all()) and float(lg.max()) < 65504.0
    if zero_q:
        assert float(lg[-1]) > 60000.0


def test_default_kv_tile_when_n_is_not_a_multiple_of_256():
    # d = 128 defaults to 256-key tiles; N = 384 is not a multiple of 256, so the default
    # must fall back to 128-key tiles (and agree with the oracle at that tile)
    import oracle
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=2, Hkv=1, N=384, bc=128)
    q, k, v = gen.inputs(w)
    qq, kq, vq, _ = gc.gpu_quantize(w, q, k, v, None, None)
    st = hifa4.new_status("cuda")
    o0, m0, l0 = hifa4.hifa4_attn_fwd_quantized(qq, kq, vq, causal=True, kv_tile=0, status=st)
    o1, m1, l1 = hifa4.hifa4_attn_fwd_quantized(qq, kq, vq, causal=True, kv_tile=128, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16)) and torch.equal(m0, m1) and torch.equal(l0, l1)
    qz = oracle.quantize_all(q, k, v)
    rows = np.arange(w.B * w.Hq * w.N, dtype=np.int64)
    ref = oracle.attn_fwd(qz, True, 128, rows)
    gc.assert_parity(gc.compare_outputs(w, rows, o0, m0, l0, ref))


@pytest.mark.parametrize("kv_tile", [64, 128])
def test_worked_examples_from_the_golden_fixture(kv_tile):
    # the hand-derived attention cases of tests/golden/worked_examples.txt on the GPU:
    # Q = 0 over a V that quantises exactly gives m = 0, l = 264 and O = 0.09375 * 2^-(c%4)
    # on every row; the first causal row gives l = 1.03125 and O = V[0]
    from tests import _golden
    G = _golden.load()
    q, k, v, vf = _golden.attn_inputs()
    qq, kq, vq, vt = gc.gpu_quantize(configs.scaled(configs.get("tiny"), N=256, d=64, bc=kv_tile), q, k, v, None,
                                     None)
    bits = lambda t: t.reshape(t.shape[0] * t.shape[1] * t.shape[2], -1).view(torch.int16).cpu().numpy().view(np.uint16)
    st = hifa4.new_status("cuda")
    o, m, l = hifa4.hifa4_attn_fwd(qq, kq, vt, causal=False, kv_tile=kv_tile, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    sec = G["attn_q_zero"]
    assert np.all(bits(m[..., None]) == _golden.num(sec["m_fp16"][0]))
    assert np.all(bits(l[..., None]) == _golden.num(sec["l_fp16"][0]))
    want = np.array([_golden.num(b) for b in sec["o_bf16_by_c_mod_4"]], np.uint16)[np.arange(64) % 4]
    assert np.all(bits(o) == want[None, :])
    o, m, l = hifa4.hifa4_attn_fwd(qq, kq, vt, causal=True, kv_tile=kv_tile, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    sec = G["attn_causal_row0"]
    assert bits(m[..., None])[0, 0] == _golden.num(sec["m_fp16"][0])
    assert bits(l[..., None])[0, 0] == _golden.num(sec["l_fp16"][0])
    o0 = o[0, 0, 0].float().cpu().numpy()
    assert o0[:16].tolist() == [float(x) for x in sec["o_first_16"]]
    assert np.array_equal(o0, vf[0].astype(np.float32))


@pytest.mark.parametrize("kv_tile", [64, 128])
def test_selected_keys_worked_example_from_the_golden_fixture(kv_tile):
    # the fixture's attn_select case: nonzero scores (S = 0 or -36) through both 4-bit
    # GEMMs; P_hat = 1.03125 on every fourth key and 0 elsewhere, l = 66, O exact in bf16
    from tests import _golden
    sec = _golden.load()["attn_select"]
    q, k, v, _ = _golden.select_inputs()
    qq, kq, vq, vt = gc.gpu_quantize(None, q, k, v, None, None)
    st = hifa4.new_status("cuda")
    o, m, l = hifa4.hifa4_attn_fwd(qq, kq, vt, causal=False, kv_tile=kv_tile, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    u16 = lambda t: t.reshape(t.shape[2], -1).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(u16(m[..., None]) == _golden.num(sec["m_fp16"][0]))
    assert np.all(u16(l[..., None]) == _golden.num(sec["l_fp16"][0]))
    want = np.array([_golden.num(b) for b in sec["o_bf16_by_c_mod_4"]], np.uint16)[np.arange(64) % 4]
    assert np.all(u16(o) == want[None, :])
