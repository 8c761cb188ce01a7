"""ctypes marshalling for the C oracle (liboracle.so).  TEST INFRASTRUCTURE ONLY.

Plain layouts used by every function here (numpy uint8 / uint16 / float arrays):
  Q/K codes  [B, H, N, d/2]   two E2M1 codes per byte, element 2i in the low nibble
  Q/K scales [B, H, N, d/16]  unsigned E4M3, one per 16 consecutive channels
  V^T codes  [B, Hkv, d, N/2] blocks of 16 consecutive tokens of one channel
  V^T scales [B, Hkv, d, N/16]
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hifa4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Which fp32 accumulation model of the 4-bit MMA the mirror uses for S (see s_dot() in
# hifa4_oracle.c): 3 = per 64-wide MMA step, acc = RZ(acc + exact sum of the step's four
# block products).  Fixed from the accumulation probe on the GPU.
S_MODEL_DEFAULT = 3

STATE_MIRROR, STATE_F64 = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no fp contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i, ll, sz, dbl = ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t, ctypes.c_double
        L.or_e2m1_encode.argtypes = [P, sz, P]
        L.or_e4m3_encode.argtypes = [P, sz, P]
        L.or_exp2.argtypes = [P, sz, P]
        L.or_quant_blocks.argtypes = [P, sz, P, P]
        L.or_e2m1_value.argtypes = [ctypes.c_uint8]
        L.or_e2m1_value.restype = ctypes.c_float
        L.or_e4m3_value.argtypes = [ctypes.c_uint8]
        L.or_e4m3_value.restype = ctypes.c_float
        L.or_calibrate.argtypes = [P, P, i, i, i, i, i, dbl, P, P]
        L.or_quantize_rows.argtypes = [P, i, i, i, i, i, P, P, P]
        L.or_quantize_vt.argtypes = [P, i, i, i, i, P, P]
        L.or_rope_rows.argtypes = [P, i, i, i, i, P, P, P]
        L.or_attn_decode.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, i, i, i, P, P, P, P, P]
        L.or_attn_decode.restype = i
        L.or_quantize_rows_f32.argtypes = [P, i, i, i, i, i, P, P, P]
        L.or_qk_scores.argtypes = [P, P, P, P, i, i, i, i, P]
        L.or_attn_fwd.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, i, i, i, i, i, P, ll, P, P, P, P]
        L.or_attn_fwd.restype = i
        L.or_attn_loop_exact.argtypes = [P, P, P, i, i, i, i, i, i, i, P, ll, P]
        L.or_attn_loop_exact.restype = i
        L.or_attn_trace.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, i, i, i, i, i, ll, P, P, P, P, P]
        L.or_attn_trace.restype = i
        L.or_attn_bruteforce.argtypes = [P, P, P, i, i, i, i, i, i, P, ll, P]
        L.or_f16_bits.argtypes = [ctypes.c_float]
        L.or_f16_bits.restype = ctypes.c_uint16
        L.or_num_threads.restype = i
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def num_threads() -> int:
    return lib().or_num_threads()


# ---------------------------------------------------------------- formats

def e2m1_encode(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().or_e2m1_encode(_p(x), x.size, _p(out))
    return out


def e4m3_encode(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().or_e4m3_encode(_p(x), x.size, _p(out))
    return out


def e2m1_value(code: int) -> float:
    return lib().or_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return lib().or_e4m3_value(code)


def exp2(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.float32)
    lib().or_exp2(_p(x), x.size, _p(out))
    return out


def quant_blocks(x):
    """Quantise a flat fp32 vector (len % 16 == 0) block by block -> (codes, scales)."""
    x = _c(x, np.float32).ravel()
    codes = np.empty(x.size // 2, np.uint8)
    scales = np.empty(x.size // 16, np.uint8)
    lib().or_quant_blocks(_p(x), x.size, _p(codes), _p(scales))
    return codes, scales


def f16_bits(x: float) -> int:
    return lib().or_f16_bits(x)


# ---------------------------------------------------------------- method steps

def calibrate(qcal, kcal, alpha):
    """Smooth-QK scales s, s^-1 [Hkv, d] from bf16 calibration tensors (uint16 bits)."""
    qcal, kcal = _c(qcal, np.uint16), _c(kcal, np.uint16)
    B, Hq, N, d = qcal.shape
    Hkv = kcal.shape[1]
    s = np.empty((Hkv, d), np.float32)
    sinv = np.empty((Hkv, d), np.float32)
    lib().or_calibrate(_p(qcal), _p(kcal), B, Hq, Hkv, N, d, float(alpha), _p(s), _p(sinv))
    return s, sinv


def quantize_rows(x, Hkv, scale=None):
    """Q or K (bf16 bits [B,H,N,d]) times an optional per-(group, channel) scale, quantised
    along d -> codes [B,H,N,d/2], scales [B,H,N,d/16]."""
    x = _c(x, np.uint16)
    B, H, N, d = x.shape
    codes = np.empty((B, H, N, d // 2), np.uint8)
    scales = np.empty((B, H, N, d // 16), np.uint8)
    sc = None if scale is None else _c(scale, np.float32)
    lib().or_quantize_rows(_p(x), B, H, Hkv, N, d, _p(sc), _p(codes), _p(scales))
    return codes, scales


def rope_rows(x, cos, sin):
    """Rotate-half RoPE of bf16 bits [B,H,N,d] with fp32 angle tables cos, sin [N, d/2]
    (row n = position of token n), in fp32 with each product and sum rounded once."""
    x = _c(x, np.uint16)
    B, H, N, d = x.shape
    cos = _c(cos, np.float32)
    sin = _c(sin, np.float32)
    assert cos.shape == (N, d // 2) and sin.shape == (N, d // 2)
    out = np.empty((B, H, N, d), np.float32)
    lib().or_rope_rows(_p(x), B, H, N, d, _p(cos), _p(sin), _p(out))
    return out


def quantize_rows_f32(x, Hkv, scale=None):
    """quantize_rows on fp32 inputs [B,H,N,d]."""
    x = _c(x, np.float32)
    B, H, N, d = x.shape
    codes = np.empty((B, H, N, d // 2), np.uint8)
    scales = np.empty((B, H, N, d // 16), np.uint8)
    sc = None if scale is None else _c(scale, np.float32)
    lib().or_quantize_rows_f32(_p(x), B, H, Hkv, N, d, _p(sc), _p(codes), _p(scales))
    return codes, scales


def quantize_rows_rope(x_pre, Hkv, cos, sin, scale=None):
    """The fused entry point: RoPE (rope_rows), then Smooth-QK and the 4-bit quantiser."""
    return quantize_rows_f32(rope_rows(x_pre, cos, sin), Hkv, scale)


def quantize_vt(v):
    v = _c(v, np.uint16)
    B, Hkv, N, d = v.shape
    codes = np.empty((B, Hkv, d, N // 2), np.uint8)
    scales = np.empty((B, Hkv, d, N // 16), np.uint8)
    lib().or_quantize_vt(_p(v), B, Hkv, N, d, _p(codes), _p(scales))
    return codes, scales


def qk_scores(qc, qs, kc, ks, model=S_MODEL_DEFAULT):
    """S [M, Nk] of one head: qc [M, d/2], qs [M, d/16], kc [Nk, d/2], ks [Nk, d/16]."""
    qc, qs, kc, ks = (_c(a, np.uint8) for a in (qc, qs, kc, ks))
    M, Nk, d = qc.shape[0], kc.shape[0], qc.shape[1] * 2
    S = np.empty((M, Nk), np.float32)
    lib().or_qk_scores(_p(qc), _p(qs), _p(kc), _p(ks), M, Nk, d, model, _p(S))
    return S


class Quantized:
    """The three quantised operands of one attention call (plain layouts)."""

    def __init__(self, qc, qs, kc, ks, vc, vs):
        self.qc, self.qs, self.kc, self.ks, self.vc, self.vs = (_c(a, np.uint8) for a in (qc, qs, kc, ks, vc, vs))
        self.B, self.Hq, self.N = qc.shape[0], qc.shape[1], qc.shape[2]
        self.Hkv = kc.shape[1]
        self.d = qc.shape[3] * 2


def quantize_all(q, k, v, s=None, sinv=None):
    """Smooth-QK (when s is given), then Q, K along d and V^T along tokens."""
    Hkv = k.shape[1]
    qc, qs = quantize_rows(q, Hkv, s)
    kc, ks = quantize_rows(k, Hkv, sinv)
    vc, vs = quantize_vt(v)
    return Quantized(qc, qs, kc, ks, vc, vs)


def attn_fwd(qz: Quantized, causal, bc, rows=None, state=STATE_MIRROR, l_from_p=False,
             s_model=S_MODEL_DEFAULT, want_f64=False, two_level=False):
    """Quantised online attention over the selected rows (all rows when rows is None).
    two_level selects the two-level P scale (a per-row, per-tile power of two under the
    block scales of P).  Returns dict with o_bf16 [n, d] (uint16), m, l [n] (fp32 holding
    the state values), m16 / l16 (fp16 bit patterns) and, when want_f64, o_f64 [n, d]."""
    n = qz.B * qz.Hq * qz.N if rows is None else len(rows)
    r = None if rows is None else _c(rows, np.int64)
    d = qz.d
    o16 = np.empty((n, d), np.uint16)
    o64 = np.empty((n, d), np.float64) if want_f64 else None
    m = np.empty(n, np.float32)
    l = np.empty(n, np.float32)
    rc = lib().or_attn_fwd(_p(qz.qc), _p(qz.qs), _p(qz.kc), _p(qz.ks), _p(qz.vc), _p(qz.vs),
                           qz.B, qz.Hq, qz.Hkv, qz.N, d, int(causal), bc, state, int(l_from_p), int(two_level),
                           s_model, _p(r), n, _p(o64), _p(o16), _p(m), _p(l))
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    out = {"o_bf16": o16, "m": m, "l": l,
           "m16": m.astype(np.float16).view(np.uint16), "l16": l.astype(np.float16).view(np.uint16)}
    if want_f64:
        out["o_f64"] = o64
    return out


def pack_decode_q(q, Hkv):
    """Decode rows of bf16 bits Q [B, Hq, nq, d] packed per kv head: [B, Hkv, 128, d], row
    r = hi * nq + t = token t of query head g * G + hi (G = Hq / Hkv); rows >= G * nq zero."""
    q = _c(q, np.uint16)
    B, Hq, nq, d = q.shape
    G = Hq // Hkv
    assert G * nq <= 128
    out = np.zeros((B, Hkv, 128, d), np.uint16)
    out[:, :, : G * nq] = q.reshape(B, Hkv, G * nq, d)
    return out


def attn_decode(qc, qs, kc, ks, vc, vs, G, nq, bc, nsplit, s_model=S_MODEL_DEFAULT):
    """Decode / split-KV attention on the packed Q_hat (codes [B, Hkv, 128, d/2], scales
    [B, Hkv, 128, d/16]) and K_hat, V_hat^T of Nk keys; see or_attn_decode.  Returns
    dict o_bf16 [B, Hkv*G, nq, d] (uint16), m, l [B, Hkv*G, nq], part_o, part_ml."""
    qc, qs, kc, ks, vc, vs = (_c(a, np.uint8) for a in (qc, qs, kc, ks, vc, vs))
    B, Hkv, R, half = qc.shape
    d = 2 * half
    Nk = kc.shape[2]
    assert R == 128
    o = np.empty((B, Hkv * G, nq, d), np.uint16)
    m = np.empty((B, Hkv * G, nq), np.float32)
    l = np.empty((B, Hkv * G, nq), np.float32)
    po = np.zeros((B * Hkv, nsplit, 128, d), np.float32)
    pml = np.zeros((B * Hkv, nsplit, 128, 2), np.float32)
    rc = lib().or_attn_decode(_p(qc), _p(qs), _p(kc), _p(ks), _p(vc), _p(vs), B, Hkv, G, nq, Nk, d, bc, nsplit,
                              s_model, _p(o), _p(m), _p(l), _p(po), _p(pml))
    if rc != 0:
        raise ValueError("oracle rejected the decode shape")
    return {"o_bf16": o, "m": m, "l": l, "part_o": po, "part_ml": pml}


def attn_trace(qz: Quantized, causal, bc, row, state=STATE_MIRROR, l_from_p=False, s_model=S_MODEL_DEFAULT,
               two_level=False):
    """Per-tile trace of one row: m after each tile, P and dequantised P_hat per key,
    O / l in the state precision, final (m, l)."""
    i = row % qz.N
    ntiles = i // bc + 1 if causal else qz.N // bc
    tr_m = np.empty(ntiles, np.float32)
    tr_p = np.empty(ntiles * bc, np.float32)
    tr_ph = np.empty(ntiles * bc, np.float32)
    o = np.empty(qz.d, np.float64)
    ml = np.empty(2, np.float32)
    rc = lib().or_attn_trace(_p(qz.qc), _p(qz.qs), _p(qz.kc), _p(qz.ks), _p(qz.vc), _p(qz.vs),
                             qz.B, qz.Hq, qz.Hkv, qz.N, qz.d, int(causal), bc, state, int(l_from_p),
                             int(two_level), s_model, int(row), _p(tr_m), _p(tr_p), _p(tr_ph), _p(o), _p(ml))
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return {"m": tr_m, "p": tr_p.reshape(ntiles, bc), "phat": tr_ph.reshape(ntiles, bc),
            "o": o, "m_final": float(ml[0]), "l_final": float(ml[1])}


def attn_loop_exact(q, k, v, causal, bc, rows=None):
    """The online tile loop with quantisation off and fp64 state."""
    q, k, v = (_c(a, np.uint16) for a in (q, k, v))
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    n = B * Hq * N if rows is None else len(rows)
    r = None if rows is None else _c(rows, np.int64)
    o = np.empty((n, d), np.float64)
    rc = lib().or_attn_loop_exact(_p(q), _p(k), _p(v), B, Hq, Hkv, N, d, int(causal), bc, _p(r), n, _p(o))
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return o


def attn_bruteforce(q, k, v, causal, rows=None):
    """Textbook softmax(QK^T/sqrt(d))V in fp64 on bf16 inputs."""
    q, k, v = (_c(a, np.uint16) for a in (q, k, v))
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    n = B * Hq * N if rows is None else len(rows)
    r = None if rows is None else _c(rows, np.int64)
    o = np.empty((n, d), np.float64)
    lib().or_attn_bruteforce(_p(q), _p(k), _p(v), B, Hq, Hkv, N, d, int(causal), _p(r), n, _p(o))
    return o
