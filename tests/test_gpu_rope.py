"""GPU parity of the fused RoPE + Smooth-QK + quantise entry point
(hifa4_quantize_qk_rope) against the oracle's rope_rows + quantiser: codes and scale
atoms bit-exact, for every head dim, with and without Smooth-QK; equality with the
unfused kernel when the rotation is exact; the attention on fused-quantised inputs."""
import numpy as np
import pytest
import torch

import oracle
from bit_flashattention_b200 import configs, gen, hifa4
from tests import _layout
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


def _pre_rope(rng, B, H, N, d, outliers=0):
    x = rng.standard_normal((B, H, N, d)).astype(np.float32)
    if outliers:
        ch = rng.choice(d, outliers, replace=False)
        x[..., ch] *= np.float32(8.0)
    return gen.f32_to_bf16_bits(x)


def _check_rows(qt, codes, scales, B, H, N, d):
    got = qt.codes.cpu().numpy().reshape(codes.shape)
    bad = np.argwhere(got != codes)
    assert bad.size == 0, (len(bad), bad[:8].tolist(), got[tuple(bad[:4].T)].tolist(), codes[tuple(bad[:4].T)].tolist())
    gs = _layout.rows_scales_to_plain(qt.scales.cpu().numpy(), B, H, N, d)
    bad = np.argwhere(gs != scales)
    assert bad.size == 0, (len(bad), bad[:8].tolist())


@pytest.mark.parametrize("d,smooth", [(64, False), (128, True), (128, False), (256, True)])
def test_fused_rope_quantiser_bit_exact(d, smooth):
    rng = np.random.default_rng(100 + d)
    B, Hq, Hkv, N = 2, 4, 2, 256
    q = _pre_rope(rng, B, Hq, N, d)
    k = _pre_rope(rng, B, Hkv, N, d, outliers=4)
    cos, sin = hifa4.hifa4_rope_table(1e6 if d == 128 else 1e4, N, d, pos0=5)
    s = sinv = None
    if smooth:
        s = (np.exp2(rng.uniform(-2, 2, (Hkv, d)))).astype(np.float32)
        sinv = (np.float32(1.0) / s).astype(np.float32)
    st = hifa4.new_status("cuda")
    qq, kq = hifa4.hifa4_quantize_qk_rope(gc.bf16_dev(q), gc.bf16_dev(k), gc.to_dev(cos), gc.to_dev(sin),
                                          None if s is None else gc.to_dev(s),
                                          None if sinv is None else gc.to_dev(sinv), status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    qc, qs = oracle.quantize_rows_rope(q, Hkv, cos, sin, s)
    kc, ks = oracle.quantize_rows_rope(k, Hkv, cos, sin, sinv)
    _check_rows(qq, qc, qs, B, Hq, N, d)
    _check_rows(kq, kc, ks, B, Hkv, N, d)


def test_fused_equals_unfused_on_exact_rotations():
    # quarter-turn angles make the rotated tensor exactly representable in bf16: the fused
    # kernel on the pre-RoPE tensor must equal the unfused kernel on the rotated one
    rng = np.random.default_rng(7)
    B, Hq, Hkv, N, d = 1, 4, 1, 128, 128
    q = _pre_rope(rng, B, Hq, N, d)
    k = _pre_rope(rng, B, Hkv, N, d, outliers=3)
    turn = rng.integers(0, 4, (N, d // 2))
    cos = np.choose(turn, [1.0, 0.0, -1.0, 0.0]).astype(np.float32)
    sin = np.choose(turn, [0.0, 1.0, 0.0, -1.0]).astype(np.float32)

    def rotate(bits):
        xf = gen.bf16_bits_to_f32(bits)
        x1, x2 = xf[..., : d // 2], xf[..., d // 2:]
        return gen.f32_to_bf16_bits(np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], -1).astype(np.float32))

    st = hifa4.new_status("cuda")
    fq, fk = hifa4.hifa4_quantize_qk_rope(gc.bf16_dev(q), gc.bf16_dev(k), gc.to_dev(cos), gc.to_dev(sin), status=st)
    uq, uk = hifa4.hifa4_quantize_qk(gc.bf16_dev(rotate(q)), gc.bf16_dev(rotate(k)), status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    for a, b in ((fq, uq), (fk, uk)):
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)


def test_attention_on_fused_quantised_inputs():
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=4, Hkv=2, N=512)
    rng = np.random.default_rng(11)
    q = _pre_rope(rng, w.B, w.Hq, w.N, w.d)
    k = _pre_rope(rng, w.B, w.Hkv, w.N, w.d, outliers=8)
    _, _, v = gen.inputs(w)
    cos, sin = hifa4.hifa4_rope_table(w.rope_theta, w.N, w.d)
    st = hifa4.new_status("cuda")
    qq, kq = hifa4.hifa4_quantize_qk_rope(gc.bf16_dev(q), gc.bf16_dev(k), gc.to_dev(cos), gc.to_dev(sin), status=st)
    vt_dev = gc.bf16_dev(v)
    o, m, l, code = gc.gpu_attention(w, qq, kq, vt_dev)
    assert code == hifa4.OK, hifa4.status_string(code)
    qc, qs = oracle.quantize_rows_rope(q, w.Hkv, cos, sin)
    kc, ks = oracle.quantize_rows_rope(k, w.Hkv, cos, sin)
    vc, vs = oracle.quantize_vt(v)
    qz = oracle.Quantized(qc, qs, kc, ks, vc, vs)
    rows = np.arange(w.B * w.Hq * w.N, dtype=np.int64)
    ref = oracle.attn_fwd(qz, w.causal, w.bc, rows)
    gc.assert_parity(gc.compare_outputs(w, rows, o, m, l, ref))


def test_fused_rope_rejects_bad_tables():
    # the binding checks the tables' type, shape and placement before the call (the C
    # ABI's own check of null tables is a CPU test)
    q = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        hifa4.hifa4_quantize_qk_rope(q, q, None, None)
    cos, sin = hifa4.hifa4_rope_table(1e4, 128, 128)
    with pytest.raises(ValueError):     # host tables
        hifa4.hifa4_quantize_qk_rope(q, q, torch.from_numpy(cos), torch.from_numpy(sin))
    with pytest.raises(ValueError):     # tables of another length
        hifa4.hifa4_quantize_qk_rope(q, q, gc.to_dev(cos[:64]), gc.to_dev(sin[:64]))


def test_exact_cancellations_give_positive_zero():
    # cos = sin = 0.5 and x_{i+d/2} = -x_i make both rotated channels cancel exactly: the
    # rounded products are equal and opposite, so the rotated values are +0 and code 0x0
    # (a fused multiply-add would leave a signed residue and could give -0, code 0x8)
    rng = np.random.default_rng(31)
    B, H, N, d = 1, 2, 128, 128
    x = rng.standard_normal((B, H, N, d // 2)).astype(np.float32)
    pre = gen.f32_to_bf16_bits(np.concatenate([x, -x], axis=-1))
    cos = np.full((N, d // 2), 0.5, np.float32)
    sin = np.full((N, d // 2), 0.5, np.float32)
    st = hifa4.new_status("cuda")
    qq, _ = hifa4.hifa4_quantize_qk_rope(gc.bf16_dev(pre), gc.bf16_dev(pre[:, :1].copy()), gc.to_dev(cos),
                                         gc.to_dev(sin), status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    qc, qs = oracle.quantize_rows_rope(pre, 1, cos, sin)
    assert np.array_equal(qq.codes.cpu().numpy().reshape(qc.shape), qc)
    # first half: RN(x c) - RN(-x s) = x, second half: RN(-x c) + RN(x s) = +0 exactly
    assert np.all(qc[..., d // 4:] == 0)
