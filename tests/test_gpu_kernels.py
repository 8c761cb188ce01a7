"""GPU checks of the building blocks through the C ABI: the device conversions and exp2,
the quantisers (bit-exact against the oracle), Smooth-QK calibration, and single-tile
probes of the block-scaled FP4 tensor-core MMAs (the S accumulation probe fixes which
fp32 accumulation model the oracle mirrors)."""
import numpy as np
import pytest
import torch

import oracle
from bit_flashattention_b200 import configs, gen, hifa4, hifa4_testhooks as th
from tests import _layout, gpu_common as gc
from tests.test_oracle_formats import _boundary_values

pytestmark = pytest.mark.gpu


def test_device_codec_and_exp2_match_oracle():
    x = _boundary_values()
    rng = np.random.default_rng(11)
    ex = np.concatenate([rng.uniform(-130, 1, 3_000_000).astype(np.float32),
                         np.arange(0xBF800000, 0xC0000000, 37, dtype=np.uint32).view(np.float32),
                         np.array([-np.inf, -127.0, -126.0, 0.0, -0.0, np.nan], np.float32)])
    allx = np.concatenate([x, ex]).astype(np.float32)
    e2, e4, e = th.probe_codec(gc.to_dev(allx))
    e2, e4, e = e2.cpu().numpy(), e4.cpu().numpy(), e.cpu().numpy()
    n = len(x)
    assert np.array_equal(e2[:n], oracle.e2m1_encode(x))
    ax = np.abs(x)
    fin = np.isfinite(ax)
    assert np.array_equal(e4[:n][fin], oracle.e4m3_encode(ax[fin]))
    assert np.array_equal(e[n:].view(np.uint32), oracle.exp2(ex).view(np.uint32))


def test_device_codec_exhaustive_over_every_finite_fp32():
    # every finite fp32 bit pattern (both signs) through the device E2M1 conversion, and every
    # finite non-negative one through the E4M3 conversion of the block scales, against the
    # oracle's codec, in chunks of 2^28 patterns.  NaN and infinity are left out: the
    # quantisers flag non-finite inputs instead of converting them, and the softmax weights
    # are finite by construction.
    chunk = 1 << 28
    e2 = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    e4 = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    checked = 0
    for start in range(0, 1 << 32, chunk):
        g2, g4 = th.probe_codec_range(start, chunk, e2, e4)
        g2, g4 = g2.cpu().numpy(), g4.cpu().numpy()
        bits = np.arange(start, start + chunk, dtype=np.uint32)
        x = bits.view(np.float32)
        fin = np.isfinite(x)
        ref2 = oracle.e2m1_encode(x[fin])
        bad = np.flatnonzero(g2[fin] != ref2)
        assert bad.size == 0, ("e2m1", [hex(int(b)) for b in bits[fin][bad[:5]]])
        if start < 0x80000000:                       # |x| of the negative half repeats these
            ref4 = oracle.e4m3_encode(x[fin])
            bad = np.flatnonzero(g4[fin] != ref4)
            assert bad.size == 0, ("e4m3", [hex(int(b)) for b in bits[fin][bad[:5]]])
        checked += int(fin.sum())
    assert checked == (1 << 32) - 2 * ((1 << 23) * 1)      # all but the 2 * 2^23 NaN/inf patterns


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("qwen3-8b-4k", dict(Hq=8, Hkv=2, N=512)),
    ("gemma2-9b-8k", dict(Hq=4, Hkv=2, N=512)),
    ("llama3.1-8b-b4-16k", dict(B=2, Hq=4, Hkv=2, N=256)),
])
def test_quantisers_bit_exact(name, kw):
    w = configs.scaled(configs.get(name), **kw)
    q, k, v = gen.inputs(w)
    s, sinv = gc.smooth_scales(w)
    qq, kq, vq, _ = gc.gpu_quantize(w, q, k, v, s, sinv)
    qz = oracle.quantize_all(q, k, v, s, sinv)
    res = gc.oracle_from_gpu_layout_check(w, qq, kq, vq, qz)
    assert all(res.values()), res


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("qwen3-8b-4k", dict(Hq=8, Hkv=2, N=512)),
    ("gemma2-9b-8k", dict(Hq=4, Hkv=2, N=256)),
    ("llama3.1-8b-b4-16k", dict(B=2, Hq=4, Hkv=2, N=256)),
])
def test_quantize_qkv_one_launch_bit_exact(name, kw):
    w = configs.scaled(configs.get(name), **kw)
    q, k, v = gen.inputs(w)
    s, sinv = gc.smooth_scales(w)
    st = hifa4.new_status("cuda")
    qq, kq, vq = hifa4.hifa4_quantize_qkv(gc.bf16_dev(q), gc.bf16_dev(k), gc.bf16_dev(v),
                                          None if s is None else gc.to_dev(s), None if sinv is None else gc.to_dev(sinv),
                                          status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    qz = oracle.quantize_all(q, k, v, s, sinv)
    res = gc.oracle_from_gpu_layout_check(w, qq, kq, vq, qz)
    assert all(res.values()), res


def test_quantisers_bit_exact_full_qwen():
    w = configs.get("qwen3-8b-4k")
    q, k, v = gen.inputs(w)
    s, sinv = gc.smooth_scales(w)
    qq, kq, vq, _ = gc.gpu_quantize(w, q, k, v, s, sinv)
    qz = oracle.quantize_all(q, k, v, s, sinv)
    res = gc.oracle_from_gpu_layout_check(w, qq, kq, vq, qz)
    assert all(res.values()), res


def test_quantize_strided_views():
    # Q as a permuted view of a [B, N, H, d] buffer (head stride d, token stride H*d)
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=4, Hkv=2, N=256)
    q, k, v = gen.inputs(w)
    qt = gc.bf16_dev(np.ascontiguousarray(q.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
    kt = gc.bf16_dev(np.ascontiguousarray(k.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
    assert not qt.is_contiguous()
    st = hifa4.new_status("cuda")
    qq, kq = hifa4.hifa4_quantize_qk(qt, kt, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    qc, qs = oracle.quantize_rows(q, w.Hkv)
    assert np.array_equal(qq.codes.cpu().numpy().reshape(qc.shape), qc)
    assert np.array_equal(_layout.rows_scales_to_plain(qq.scales.cpu().numpy(), w.B, w.Hq, w.N, w.d), qs)


def test_nonfinite_input_is_flagged():
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=2, Hkv=1, N=128)
    q, k, v = gen.inputs(w)
    q = q.copy()
    q[0, 1, 77, 5] = 0x7F80          # +inf in bf16
    st = hifa4.new_status("cuda")
    hifa4.hifa4_quantize_qk(gc.bf16_dev(q), gc.bf16_dev(k), status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.ERR_NONFINITE
    v = v.copy()
    v[0, 0, 3, 9] = 0x7FC0           # NaN
    hifa4.hifa4_quantize_v(gc.bf16_dev(v), status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.ERR_NONFINITE
    assert hifa4.hifa4_read_status(st) == hifa4.OK   # cleared


@pytest.mark.parametrize("name,kw", [("qwen3-8b-4k", dict(Hq=8, Hkv=2, N=384)),
                                     ("gemma2-9b-8k", dict(Hq=4, Hkv=2, N=300))])
def test_calibrate_matches_oracle(name, kw):
    w = configs.scaled(configs.get(name), **kw)
    qc, kc, _ = gen.inputs(w, calib=True)
    s, si = hifa4.hifa4_calibrate_smooth(gc.bf16_dev(qc), gc.bf16_dev(kc), w.alpha)
    so, sio = oracle.calibrate(qc, kc, w.alpha)
    assert np.array_equal(s.cpu().numpy(), so) and np.array_equal(si.cpu().numpy(), sio)


def _rand_tile(rng, rows, d, narrow):
    codes = rng.integers(0, 256, (rows, d // 2), dtype=np.uint8)
    lo, hi = (0x30, 0x48) if narrow else (0x01, 0x7E)
    scales = rng.integers(lo, hi + 1, (rows, d // 16), dtype=np.uint8)
    return codes, scales


def _atoms_rows(scales, rows, d):
    full = np.zeros((128, d // 16), np.uint8)
    full[:rows] = scales
    return _layout.rows_scales_from_plain(full[None, None], 1, 1, 128, d)


@pytest.mark.parametrize("d,bc", [(64, 64), (64, 128), (128, 64), (128, 128), (256, 64)])
def test_qk_mma_probe_accumulation_model(d, bc):
    rng = np.random.default_rng(d * 1000 + bc)
    counts = {}
    for narrow in (True, False):
        qc, qs = _rand_tile(rng, 128, d, narrow)
        kc, ks = _rand_tile(rng, bc, d, narrow)
        S = th.probe_qk_tile(gc.to_dev(qc), gc.to_dev(_atoms_rows(qs, 128, d)), gc.to_dev(kc),
                                      gc.to_dev(_atoms_rows(ks, bc, d)), d, bc).cpu().numpy()
        exact = oracle.qk_scores(qc, qs, kc, ks, 2).astype(np.float64)
        rel = np.max(np.abs(S - exact) / np.maximum(np.abs(exact), 1e-30))
        for model in (0, 1, 2, 3):
            ref = oracle.qk_scores(qc, qs, kc, ks, model)
            counts[(narrow, model)] = int(np.sum(S.view(np.uint32) != ref.view(np.uint32)))
        counts[(narrow, "max_rel_vs_exact")] = float(rel)
    print(f"\nQK probe d={d} bc={bc} mismatches per model (narrow scales?, model): {counts}")
    assert counts[(True, "max_rel_vs_exact")] < 1e-5 and counts[(False, "max_rel_vs_exact")] < 1e-3, counts
    assert counts[(True, oracle.S_MODEL_DEFAULT)] == 0 and counts[(False, oracle.S_MODEL_DEFAULT)] == 0, counts


@pytest.mark.parametrize("d,bc", [(64, 64), (64, 128), (128, 64), (128, 128), (256, 64)])
def test_pv_mma_probe(d, bc):
    import ml_dtypes
    rng = np.random.default_rng(7 * d + bc)
    pc = (rng.integers(0, 8, (128, bc)) | (rng.integers(0, 8, (128, bc)) << 4)).astype(np.uint8)[:, : bc // 2]
    ps = rng.integers(0x00, 0x38, (128, bc // 16), dtype=np.uint8)           # P_hat scales <= 1, incl. 0 / subnormal
    vc = rng.integers(0, 256, (d, bc // 2), dtype=np.uint8)
    vs = rng.integers(0x28, 0x48, (d, bc // 16), dtype=np.uint8)
    p_atoms = _layout.rows_scales_from_plain(ps[None, None], 1, 1, 128, bc)
    v_atoms = _layout.vt_scales_from_plain(vs[None, None], 1, 1, bc, d)
    O, R = th.probe_pv_tile(gc.to_dev(pc), gc.to_dev(p_atoms), gc.to_dev(vc), gc.to_dev(v_atoms), d, bc)
    O, R = O.cpu().numpy().astype(np.float64), R.cpu().numpy().astype(np.float64)

    def deq(c, s):
        lo = (c & 15).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        hi = (c >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        x = np.stack([lo, hi], -1).reshape(c.shape[0], -1)
        return x * np.repeat(s.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=1)

    P, V = deq(pc, ps), deq(vc, vs)
    ref = P @ V.T
    assert np.max(np.abs(O - ref)) <= 1e-5 * max(1.0, np.abs(ref).max())
    assert np.array_equal(R, P.sum(1))          # the normaliser column is exact


def test_quantize_qkv_strided_and_full_size():
    # the one-launch quantiser (TMA-fed): permuted [B, N, H, d] views of Q, K, V, and the
    # full qwen3-8b-4k tensors of the benchmark, bit-exact against the oracle
    w = configs.scaled(configs.get("qwen3-8b-4k"), B=2, Hq=4, Hkv=2, N=256)
    q, k, v = gen.inputs(w)
    views = [gc.bf16_dev(np.ascontiguousarray(x.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3) for x in (q, k, v)]
    assert not views[0].is_contiguous()
    s, sinv = gc.smooth_scales(w)
    st = hifa4.new_status("cuda")
    qq, kq, vq = hifa4.hifa4_quantize_qkv(*views, gc.to_dev(s), gc.to_dev(sinv), status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    res = gc.oracle_from_gpu_layout_check(w, qq, kq, vq, oracle.quantize_all(q, k, v, s, sinv))
    assert all(res.values()), res

    w = configs.get("qwen3-8b-4k")
    q, k, v = gen.inputs(w)
    s, sinv = gc.smooth_scales(w)
    qq, kq, vq = hifa4.hifa4_quantize_qkv(gc.bf16_dev(q), gc.bf16_dev(k), gc.bf16_dev(v), gc.to_dev(s),
                                          gc.to_dev(sinv), status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    res = gc.oracle_from_gpu_layout_check(w, qq, kq, vq, oracle.quantize_all(q, k, v, s, sinv))
    assert all(res.values()), res


def test_quantize_qkv_flags_nonfinite_input():
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=2, Hkv=1, N=256)
    q, k, v = gen.inputs(w)
    vt = gc.bf16_dev(v)
    vt[0, 0, 77, 5] = float("inf")
    st = hifa4.new_status("cuda")
    hifa4.hifa4_quantize_qkv(gc.bf16_dev(q), gc.bf16_dev(k), vt, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.ERR_NONFINITE
