"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and the
oracle on the same seeded inputs, and compare."""
import ml_dtypes
import numpy as np
import torch

import oracle
from bit_flashattention_b200 import gen, hifa4
from tests import _layout

# Tolerances on the attention output O (per the target: FP16 m and l exact, codes and
# scales bit-exact, O within these bounds).
O_MAX_ABS = 1e-2
O_MEAN_REL = 1e-3


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(bits):
    return to_dev(bits.view(np.int16)).view(torch.bfloat16)


def smooth_scales(w):
    """Oracle Smooth-QK scales of a workload (None when Smooth-QK is disabled)."""
    if w.alpha is None:
        return None, None
    qc, kc, _ = gen.inputs(w, calib=True)
    return oracle.calibrate(qc, kc, w.alpha)


def gpu_quantize(w, q, k, v, s, sinv):
    st = hifa4.new_status("cuda")
    qt, kt, vt = bf16_dev(q), bf16_dev(k), bf16_dev(v)
    s_t = None if s is None else to_dev(s)
    si_t = None if sinv is None else to_dev(sinv)
    qq, kq = hifa4.hifa4_quantize_qk(qt, kt, s_t, si_t, status=st)
    vq = hifa4.hifa4_quantize_v(vt, status=st)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    return qq, kq, vq, vt


def gpu_attention(w, qq, kq, vt_bf16):
    st = hifa4.new_status("cuda")
    o, m, l = hifa4.hifa4_attn_fwd(qq, kq, vt_bf16, causal=w.causal, kv_tile=w.bc, status=st)
    code = hifa4.hifa4_read_status(st)
    return o, m, l, code


def oracle_from_gpu_layout_check(w, qq, kq, vq, qz):
    """Bit-exact comparison of the GPU's 4-bit tensors with the oracle's (plain layouts)."""
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    res = {}
    res["q_codes"] = np.array_equal(qq.codes.cpu().numpy().reshape(qz.qc.shape), qz.qc)
    res["k_codes"] = np.array_equal(kq.codes.cpu().numpy().reshape(qz.kc.shape), qz.kc)
    res["v_codes"] = np.array_equal(vq.codes.cpu().numpy().reshape(qz.vc.shape), qz.vc)
    res["q_scales"] = np.array_equal(_layout.rows_scales_to_plain(qq.scales.cpu().numpy(), B, Hq, N, d), qz.qs)
    res["k_scales"] = np.array_equal(_layout.rows_scales_to_plain(kq.scales.cpu().numpy(), B, Hkv, N, d), qz.ks)
    res["v_scales"] = np.array_equal(_layout.vt_scales_to_plain(vq.scales.cpu().numpy(), B, Hkv, N, d), qz.vs)
    return res


def compare_outputs(w, rows, o, m, l, ref):
    """Element-wise comparison of GPU (o, m, l) at the given row ids with the oracle's."""
    d = w.d
    o_all = o.reshape(-1, d).view(torch.int16).cpu().numpy().view(np.uint16)
    m_all = m.reshape(-1).float().cpu().numpy()
    l_all = l.reshape(-1).float().cpu().numpy()
    og = o_all[rows].view(ml_dtypes.bfloat16).astype(np.float64)
    orf = ref["o_bf16"].view(ml_dtypes.bfloat16).astype(np.float64)
    mg, lg = m_all[rows], l_all[rows]
    diff = np.abs(og - orf)
    return {
        "m_mismatch": int(np.sum(mg != ref["m"])),
        "l_mismatch": int(np.sum(lg != ref["l"])),
        "rows": len(rows),
        "o_max_abs": float(diff.max()),
        "o_mean_rel": float(diff.mean() / max(np.abs(orf).mean(), 1e-30)),
        "o_finite": bool(np.all(np.isfinite(og))),
    }


def assert_parity(stats):
    assert stats["o_finite"], stats
    assert stats["m_mismatch"] == 0, stats
    assert stats["l_mismatch"] == 0, stats
    assert stats["o_max_abs"] <= O_MAX_ABS, stats
    assert stats["o_mean_rel"] <= O_MEAN_REL, stats


def run_parity(w, rows=None, check_quant=True):
    """Full path on GPU vs oracle for a workload; rows=None compares every row."""
    q, k, v = gen.inputs(w)
    s, sinv = smooth_scales(w)
    qq, kq, vq, vt = gpu_quantize(w, q, k, v, s, sinv)
    qz = oracle.quantize_all(q, k, v, s, sinv)
    if check_quant:
        res = oracle_from_gpu_layout_check(w, qq, kq, vq, qz)
        assert all(res.values()), res
    o, m, l, code = gpu_attention(w, qq, kq, vt)
    assert code == hifa4.OK, hifa4.status_string(code)
    if rows is None:
        rows = np.arange(w.B * w.Hq * w.N, dtype=np.int64)
    ref = oracle.attn_fwd(qz, w.causal, w.bc, rows)
    stats = compare_outputs(w, rows, o, m, l, ref)
    print(f"\n{w.name} B{w.B} Hq{w.Hq} Hkv{w.Hkv} N{w.N} d{w.d} bc{w.bc} causal={w.causal}: {stats}")
    return stats
