"""Pins of the oracle's online tile loop: textbook attention when quantisation is off,
the P-Reordering identity, the inconsistent formulation's coherent output scaling,
net probability-mass loss, and closed-form special cases."""
import ml_dtypes
import numpy as np
import pytest
import torch

from bit_flashattention_b200 import configs, gen


def _small(name="qwen3-8b-4k", **kw):
    return configs.scaled(configs.get(name), **kw)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bc", [16, 32])
def test_exact_loop_equals_textbook_softmax(orc, causal, bc):
    w = _small(B=2, Hq=4, Hkv=2, N=64, d=64)
    q, k, v = gen.inputs(w)
    o_loop = orc.attn_loop_exact(q, k, v, causal, bc)
    o_bf = orc.attn_bruteforce(q, k, v, causal)
    assert np.max(np.abs(o_loop - o_bf)) <= 1e-12
    # and torch's SDPA in fp64 (library routine) with the GQA expansion
    t = lambda a: torch.from_numpy(gen.bf16_bits_to_f32(a).astype(np.float64))
    kt = t(k).repeat_interleave(w.Hq // w.Hkv, dim=1)
    vt = t(v).repeat_interleave(w.Hq // w.Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), kt, vt, is_causal=causal)
    assert np.max(np.abs(o_loop - ref.reshape(-1, w.d).numpy())) <= 1e-12


def _quantized(w, smooth=True):
    q, k, v = gen.inputs(w)
    s = sinv = None
    if smooth and w.alpha is not None:
        qc_, kc_, _ = gen.inputs(w, calib=True)
        s, sinv = __import__("oracle").calibrate(qc_, kc_, w.alpha)
    return __import__("oracle").quantize_all(q, k, v, s, sinv), (q, k, v)


def _vhat(qz):
    lo = (qz.vc & 0xF).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    hi = (qz.vc >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    v = np.stack([lo, hi], -1).reshape(*qz.vc.shape[:-1], qz.vc.shape[-1] * 2)
    s = np.repeat(qz.vs.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=-1)
    return np.swapaxes(v * s, 2, 3)          # [B, Hkv, N, d]


@pytest.mark.parametrize("causal", [False, True])
def test_p_reordering_identity(orc, causal):
    # Online result with fp64 state and exact 2^x must equal the batch formula
    # O = sum_t 2^(m_t - m_T) P_hat_t V_hat / sum_t 2^(m_t - m_T) rowsum(P_hat_t).
    w = _small(Hq=2, Hkv=1, N=256, d=64)
    qz, _ = _quantized(w)
    vh = _vhat(qz)
    bc = 64
    for row in (0, 5, 63, 64, 130, 255, 256 + 200, 511):
        tr = orc.attn_trace(qz, causal, bc, row, state=orc.STATE_F64)
        mT = tr["m"][-1]
        wts = np.exp2(tr["m"].astype(np.float64) - mT)[:, None] * tr["phat"].astype(np.float64)
        h = (row // w.N) % w.Hq
        keys = wts.size
        num = wts.reshape(-1) @ vh[0, h // (w.Hq // w.Hkv), :keys]
        den = wts.sum()
        assert np.max(np.abs(tr["o"] - num / den)) <= 1e-12 * max(1.0, np.max(np.abs(num / den)))
        assert abs(tr["l_final"] - den) <= 1e-6 * den


def test_inconsistent_formulation_is_a_coherent_output_scaling(orc):
    # With the normaliser summed from unquantised P, O differs from the P-Reordering O by
    # one factor per row, the same for every channel: l_consistent / l_inconsistent.
    w = _small(Hq=2, Hkv=1, N=256, d=64)
    qz, _ = _quantized(w)
    rows = np.arange(0, 512, 7)
    a = orc.attn_fwd(qz, True, 64, rows, state=orc.STATE_F64, want_f64=True)
    b = orc.attn_fwd(qz, True, 64, rows, state=orc.STATE_F64, l_from_p=True, want_f64=True)
    ratio = (a["l"].astype(np.float64) / b["l"].astype(np.float64))[:, None]
    assert np.allclose(b["o_f64"], a["o_f64"] * ratio, rtol=1e-5, atol=1e-9)


def test_net_probability_mass_loss_sign(orc):
    # HiFA4 abstract: under the inconsistent formulation every measured attention tile
    # showed net probability-mass loss (median eps_bar < 0).  eps per row and tile =
    # sum(P_hat)/sum(P) - 1 over unmasked keys; eps_bar = mean over the tile's rows.
    w = _small(Hq=2, Hkv=1, N=512, d=128)
    qz, _ = _quantized(w)
    bc, br = 128, 128
    eps_tiles = {}
    for row in range(0, w.Hq * w.N, 3):
        tr = orc.attn_trace(qz, True, bc, row)
        sp, sph = tr["p"].astype(np.float64).sum(1), tr["phat"].astype(np.float64).sum(1)
        for j in range(len(sp)):
            if sp[j] > 0:
                eps_tiles.setdefault((row // br, j), []).append(sph[j] / sp[j] - 1)
    eps_bar = np.array([np.mean(v) for v in eps_tiles.values()])
    assert np.median(eps_bar) < 0
    assert np.mean(eps_bar < 0) > 0.9


def test_causal_first_row_is_first_value_row(orc):
    # Row 0 sees key 0 only: P = E(~0) ~ 1 -> P_hat = 6 * RN_E4M3(P/6) and l = fp16(P_hat),
    # so O_0 = bf16(V_hat[0]) exactly.
    w = _small(Hq=2, Hkv=1, N=256, d=64)
    qz, _ = _quantized(w)
    out = orc.attn_fwd(qz, True, 64, np.array([0, w.N], np.int64))
    vh = _vhat(qz)[0, 0, 0].astype(np.float32)
    ref = vh.astype(ml_dtypes.bfloat16).astype(np.float32)       # compared as values: -0 == +0
    got = out["o_bf16"].view(ml_dtypes.bfloat16).astype(np.float32)
    assert np.array_equal(got[0], ref) and np.array_equal(got[1], ref)


def test_equal_scores_give_mean_of_values(orc):
    # Q = 0 makes every score 0: P = 1 for all keys, P_hat identical, O = mean of V_hat.
    w = _small(Hq=1, Hkv=1, N=256, d=64)
    q, k, v = gen.inputs(w)
    q = np.zeros_like(q)
    qz = orc.quantize_all(q, k, v)
    out = orc.attn_fwd(qz, False, 64, np.array([3, 100], np.int64), want_f64=True)
    mean = _vhat(qz)[0, 0].mean(0)
    assert np.allclose(out["o_f64"][0], mean, rtol=1e-6, atol=1e-6)
    assert np.all(out["m"] == 0.0)
    assert np.all(out["l"] == np.float32(256 * 1.03125))


def test_mirror_close_to_exact_attention(orc):
    # The 4-bit path stays close to fp64 softmax attention on the same dequantised Q, K, V
    # (numpy, no tiles): quantising P and keeping fp16 state add little on top of the
    # operand quantisation, while a dropped or misplaced term in the loop would not.
    from tests.test_oracle_quant import _dequant
    w = _small(Hq=4, Hkv=2, N=512, d=128)
    qz, (q, k, v) = _quantized(w)
    rows = np.arange(0, w.Hq * w.N)
    ref = orc.attn_bruteforce(q, k, v, True, rows).reshape(w.Hq, w.N, w.d)
    mir = orc.attn_fwd(qz, True, 128, rows, want_f64=True)["o_f64"].reshape(w.Hq, w.N, w.d)
    qd, kd, vd = _dequant(qz.qc, qz.qs)[0].astype(np.float64), _dequant(qz.kc, qz.ks)[0].astype(np.float64), _vhat(qz)[0]
    deq = []
    for h in range(w.Hq):
        g = h // (w.Hq // w.Hkv)
        S = qd[h] @ kd[g].T / np.sqrt(w.d) + np.triu(np.full((w.N, w.N), -np.inf), 1)
        P = np.exp(S - S.max(1, keepdims=True))
        deq.append(P @ vd[g] / P.sum(1, keepdims=True))
    deq = np.stack(deq)
    rel = lambda a, b: np.abs(a - b).mean() / np.abs(b).mean()
    assert rel(mir, deq) < 0.08
    assert rel(mir, ref) < 1.2 * rel(deq, ref)
    qz0, _ = _quantized(w, smooth=False)
    direct = orc.attn_fwd(qz0, True, 128, rows, l_from_p=True, want_f64=True)["o_f64"].reshape(w.Hq, w.N, w.d)
    print(f"\nrelative error vs fp64 attention: HiFA4 {rel(mir, ref):.4f} (operand quantisation alone "
          f"{rel(deq, ref):.4f}), direct FP4 {rel(direct, ref):.4f}")


@pytest.mark.parametrize("causal", [False, True])
def test_running_max_is_the_fp16_rounding_of_the_scaled_row_max(orc, causal):
    # the online-softmax state is FP16: the final m of a row is the FP16 rounding (nearest
    # even) of the largest RN(S * c) over its visible keys, whatever the tile order, since
    # that rounding is monotone; m and l are FP16 values
    w = _small(B=1, Hq=2, Hkv=1, N=256, d=128)
    qz, _ = _quantized(w)
    ref = orc.attn_fwd(qz, causal, 64)
    c = np.float32(np.log2(np.e) / np.sqrt(w.d))
    for h in range(w.Hq):
        S = orc.qk_scores(qz.qc[0, h], qz.qs[0, h], qz.kc[0, 0], qz.ks[0, 0])
        t = (S.astype(np.float32) * c).astype(np.float32)
        if causal:
            t = np.where(np.tril(np.ones_like(t, dtype=bool)), t, -np.inf)
        want = t.max(axis=1).astype(np.float16)
        got = ref["m"][h * w.N:(h + 1) * w.N]
        assert np.array_equal(got.astype(np.float16), want)
        assert np.array_equal(got, want.astype(np.float32))
    assert np.array_equal(ref["l"], ref["l"].astype(np.float16).astype(np.float32))
