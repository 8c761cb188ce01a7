"""Thin Python binding of the C ABI in include/hifa4.h (argument marshalling only).

Every step of the attention path runs in the CUDA library libhifa4.so; this module only
allocates result tensors with torch (device memory), passes raw pointers and the current
CUDA stream, and turns status codes into exceptions.  There is no CPU fallback: if the
library is missing or the device is not an sm_100 GPU, calls raise.
"""
import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhifa4.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "hifa4.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_UNSUPPORTED_DEVICE, ERR_NONFINITE, ERR_TIMEOUT, ERR_CUDA, ERR_IO = range(8)


class Hifa4Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


class _QT(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("B", ctypes.c_int), ("H", ctypes.c_int),
                ("N", ctypes.c_int), ("d", ctypes.c_int), ("transposed", ctypes.c_int)]


_lib = None


def lib():
    """Load libhifa4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with bit_flashattention_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, i, sz, f, ull = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_ulonglong
        QP = ctypes.POINTER(_QT)
        sig = {
            "hifa4_status_string": ([i], ctypes.c_char_p),
            "hifa4_qtensor_codes_bytes": ([i, i, i, i], sz),
            "hifa4_qtensor_scales_bytes": ([i, i, i, i, i], sz),
            "hifa4_calibrate_workspace_bytes": ([i, i], sz),
            "hifa4_calibrate_smooth": ([P, P, P, P, i, i, i, i, i, f, P, P, P, P], i),
            "hifa4_quantize_qk": ([P, P, P, P, i, i, i, i, i, P, P, QP, QP, P, P], i),
            "hifa4_quantize_v": ([P, P, i, i, i, i, QP, P, P], i),
            "hifa4_quantize_qk_rope": ([P, P, P, P, i, i, i, i, i, P, P, P, P, QP, QP, P, P], i),
            "hifa4_rope_table": ([ctypes.c_double, i, i, i, P, P], i),
            "hifa4_quantize_qkv": ([P, P, P, P, P, P, i, i, i, i, i, P, P, QP, QP, QP, P, P], i),
            "hifa4_attn_fwd_quantized": ([QP, QP, QP, i, i, i, i, i, i, i, P, P, P, P, P], i),
            "hifa4_attn_fwd_quantized_fast": ([QP, QP, QP, i, i, i, i, i, i, i, P, P, P, P, P], i),
            "hifa4_attn_fwd_ablation": ([QP, QP, QP, i, i, i, i, i, i, i, i, i, P, P, P, P, P, P], i),
            "hifa4_quantize_q_decode": ([P, P, i, i, i, i, i, P, QP, P, P], i),
            "hifa4_decode_workspace_bytes": ([i, i, i, i], sz),
            "hifa4_attn_decode": ([QP, QP, QP, i, i, i, i, i, i, i, i, P, sz, P, P, P, P, P], i),
            "hifa4_attn_workspace_bytes": ([i, i, i, i], sz),
            "hifa4_attn_fwd": ([QP, QP, P, P, i, i, i, i, i, i, i, P, sz, P, P, P, P, P], i),
            "hifa4_read_status": ([P, i, P], i),
            "hifa4_set_wait_limit_ns": ([ull], None),
            "hifa4_calibration_save": ([ctypes.c_char_p, i, i, f, P, P], i),
            "hifa4_calibration_load": ([ctypes.c_char_p, P, P, P, P, P, sz], i),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def declared_functions(header=HEADER_PATH):
    """Names of the functions a header of this library (default include/hifa4.h) declares."""
    txt = open(header).read()
    return sorted(set(re.findall(r"HIFA4_API\s+[\w\s\*]+?\b(hifa4_\w+)\s*\(", txt)))


def status_string(code: int) -> str:
    return lib().hifa4_status_string(code).decode()


def _check(code: int, what: str):
    if code != OK:
        raise Hifa4Error(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, what, shape=None, contiguous=False):
    """Raise unless `t` is a CUDA tensor of `dtype` (and `shape`, and contiguous when
    asked): the library takes raw device pointers and cannot tell a host buffer or a
    tensor of another type from the one it expects."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype is not dtype:
        raise TypeError(f"{what}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{what}: must be on a CUDA device, is on {t.device}")
    if shape is not None and t.shape != shape:
        raise ValueError(f"{what}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")
    return t


def _need_opt(t, dtype, what, shape=None):
    return None if t is None else _need(t, dtype, what, shape, contiguous=True)


def _need_qt(t, what):
    # a QTensor's buffers are checked when it is built
    if not isinstance(t, QTensor):
        raise TypeError(f"{what}: expected a QTensor, got {type(t).__name__}")
    return t


def _smooth(s, sinv, Hkv, d):
    _need_opt(s, torch.float32, "s", (Hkv, d))
    _need_opt(sinv, torch.float32, "sinv", (Hkv, d))


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _strides(x):
    s = x.stride()
    if s[3] != 1:
        raise ValueError("the channel dimension must be contiguous")
    return (ctypes.c_int64 * 3)(s[0], s[1], s[2])


class QTensor:
    """A 4-bit tensor in the library's layout: uint8 `codes` and `scales` on the GPU."""

    def __init__(self, B, H, N, d, transposed, device=None, codes=None, scales=None):
        self.B, self.H, self.N, self.d, self.transposed = B, H, N, d, int(transposed)
        L = lib()
        nc = L.hifa4_qtensor_codes_bytes(B, H, N, d)
        ns = L.hifa4_qtensor_scales_bytes(B, H, N, d, self.transposed)
        self.codes = codes if codes is not None else torch.empty(nc, dtype=torch.uint8, device=device)
        self.scales = scales if scales is not None else torch.empty(ns, dtype=torch.uint8, device=device)
        for t, w, n in ((self.codes, "codes", nc), (self.scales, "scales", ns)):
            _need(t, torch.uint8, "QTensor." + w, contiguous=True)
            if t.numel() < n:
                raise ValueError(f"QTensor.{w}: {t.numel()} bytes, the layout needs {n}")

    def c(self):
        return ctypes.byref(_QT(self.codes.data_ptr(), self.scales.data_ptr(), self.B, self.H, self.N, self.d,
                                self.transposed))


def new_status(device=None):
    return torch.zeros(1, dtype=torch.int32, device=device)


def _status(status, device):
    """The caller's device status word (int32, checked) or a new zeroed one."""
    return new_status(device) if status is None else _need(status, torch.int32, "status")


def hifa4_read_status(status, clear=True):
    _need(status, torch.int32, "status")
    return lib().hifa4_read_status(_ptr(status), int(clear), _stream())


def hifa4_set_wait_limit_ns(ns: int):
    lib().hifa4_set_wait_limit_ns(int(ns))


def hifa4_calibrate_smooth(q_cal, k_cal, alpha: float):
    """Smooth-QK scales (s, s_inv), fp32 [Hkv, d] on q_cal's device.  Synchronises."""
    _need(q_cal, torch.bfloat16, "q_cal")
    _need(k_cal, torch.bfloat16, "k_cal")
    B, Hq, N, d = q_cal.shape
    Hkv = k_cal.shape[1]
    dev = q_cal.device
    s = torch.empty(Hkv, d, dtype=torch.float32, device=dev)
    si = torch.empty_like(s)
    ws = torch.empty(lib().hifa4_calibrate_workspace_bytes(Hkv, d), dtype=torch.uint8, device=dev)
    _check(lib().hifa4_calibrate_smooth(_ptr(q_cal), _ptr(k_cal), _strides(q_cal), _strides(k_cal), B, Hq, Hkv, N, d,
                                        float(alpha), _ptr(s), _ptr(si), _ptr(ws), _stream()), "hifa4_calibrate_smooth")
    return s, si


def hifa4_calibration_save(path, s, sinv, alpha: float):
    """Write the Smooth-QK scales s, s_inv (fp32 [Hkv, d], any device) and alpha to `path`."""
    import numpy as np
    sh = np.ascontiguousarray(s.detach().float().cpu().numpy())
    sih = np.ascontiguousarray(sinv.detach().float().cpu().numpy())
    if sh.ndim != 2 or sih.shape != sh.shape:
        raise ValueError("s and sinv must both be [Hkv, d]")
    _check(lib().hifa4_calibration_save(os.fsencode(path), sh.shape[0], sh.shape[1], float(alpha),
                                        sh.ctypes.data_as(ctypes.c_void_p), sih.ctypes.data_as(ctypes.c_void_p)),
           "hifa4_calibration_save")


def hifa4_calibration_load(path, device=None):
    """Read a calibration file -> (s, s_inv fp32 [Hkv, d] on `device`, alpha)."""
    import numpy as np
    hk, dd, al = ctypes.c_int(), ctypes.c_int(), ctypes.c_float()
    _check(lib().hifa4_calibration_load(os.fsencode(path), ctypes.byref(hk), ctypes.byref(dd), ctypes.byref(al), None,
                                        None, 0), "hifa4_calibration_load")
    sh = np.empty((hk.value, dd.value), np.float32)
    sih = np.empty_like(sh)
    _check(lib().hifa4_calibration_load(os.fsencode(path), ctypes.byref(hk), ctypes.byref(dd), ctypes.byref(al),
                                        sh.ctypes.data_as(ctypes.c_void_p), sih.ctypes.data_as(ctypes.c_void_p),
                                        sh.size), "hifa4_calibration_load")
    return torch.from_numpy(sh).to(device), torch.from_numpy(sih).to(device), float(al.value)


def hifa4_quantize_qk(q, k, s=None, sinv=None, status=None, out=None):
    """Smooth-QK + 4-bit quantisation of bf16 Q [B,Hq,N,d] and K [B,Hkv,N,d] -> (QTensor, QTensor)."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    _smooth(s, sinv, Hkv, d)
    if out is None:
        out = (QTensor(B, Hq, N, d, 0, q.device), QTensor(B, Hkv, N, d, 0, q.device))
    st = _status(status, q.device)
    _check(lib().hifa4_quantize_qk(_ptr(q), _ptr(k), _strides(q), _strides(k), B, Hq, Hkv, N, d, _ptr(s), _ptr(sinv),
                                   out[0].c(), out[1].c(), _ptr(st), _stream()), "hifa4_quantize_qk")
    return out


def hifa4_rope_table(theta: float, N: int, d: int, pos0: int = 0):
    """Host fp32 angle tables (cos, sin) [N, d/2] of positions pos0..pos0+N-1 (numpy)."""
    import numpy as np
    cos = np.empty((N, d // 2), np.float32)
    sin = np.empty((N, d // 2), np.float32)
    _check(lib().hifa4_rope_table(float(theta), int(pos0), N, d, cos.ctypes.data_as(ctypes.c_void_p),
                                  sin.ctypes.data_as(ctypes.c_void_p)), "hifa4_rope_table")
    return cos, sin


def hifa4_quantize_qk_rope(q, k, rope_cos, rope_sin, s=None, sinv=None, status=None, out=None):
    """Fused RoPE + Smooth-QK + 4-bit quantisation of PRE-RoPE bf16 Q [B,Hq,N,d] and K
    [B,Hkv,N,d]; rope_cos, rope_sin: device fp32 [N, d/2] -> (QTensor, QTensor)."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    _need(rope_cos, torch.float32, "rope_cos", (N, d // 2), contiguous=True)
    _need(rope_sin, torch.float32, "rope_sin", (N, d // 2), contiguous=True)
    _smooth(s, sinv, Hkv, d)
    if out is None:
        out = (QTensor(B, Hq, N, d, 0, q.device), QTensor(B, Hkv, N, d, 0, q.device))
    st = _status(status, q.device)
    _check(lib().hifa4_quantize_qk_rope(_ptr(q), _ptr(k), _strides(q), _strides(k), B, Hq, Hkv, N, d, _ptr(rope_cos),
                                        _ptr(rope_sin), _ptr(s), _ptr(sinv), out[0].c(), out[1].c(), _ptr(st),
                                        _stream()), "hifa4_quantize_qk_rope")
    return out


def hifa4_quantize_qkv(q, k, v, s=None, sinv=None, status=None, out=None):
    """Smooth-QK + 4-bit Q, K and V^T in one launch -> (QTensor, QTensor, QTensor)."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    _need(v, torch.bfloat16, "v")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    _smooth(s, sinv, Hkv, d)
    if out is None:
        out = (QTensor(B, Hq, N, d, 0, q.device), QTensor(B, Hkv, N, d, 0, q.device), QTensor(B, Hkv, N, d, 1, q.device))
    st = _status(status, q.device)
    _check(lib().hifa4_quantize_qkv(_ptr(q), _ptr(k), _ptr(v), _strides(q), _strides(k), _strides(v), B, Hq, Hkv, N, d,
                                    _ptr(s), _ptr(sinv), out[0].c(), out[1].c(), out[2].c(), _ptr(st), _stream()),
           "hifa4_quantize_qkv")
    return out


def hifa4_quantize_v(v, status=None, out=None):
    """4-bit quantisation of V^T (blocks of 16 tokens) of bf16 V [B,Hkv,N,d] -> QTensor."""
    _need(v, torch.bfloat16, "v")
    B, Hkv, N, d = v.shape
    out = out if out is not None else QTensor(B, Hkv, N, d, 1, v.device)
    st = _status(status, v.device)
    _check(lib().hifa4_quantize_v(_ptr(v), _strides(v), B, Hkv, N, d, out.c(), _ptr(st), _stream()), "hifa4_quantize_v")
    return out


def _outputs(B, Hq, N, d, dev, o, m, l):
    """Output tensors o bf16 [B, Hq, N, d], m and l fp16 [B, Hq, N]: the given ones after
    checking them, else new ones."""
    if o is None:
        o = torch.empty(B, Hq, N, d, dtype=torch.bfloat16, device=dev)
    if m is None:
        m = torch.empty(B, Hq, N, dtype=torch.float16, device=dev)
    if l is None:
        l = torch.empty(B, Hq, N, dtype=torch.float16, device=dev)
    _need(o, torch.bfloat16, "o", (B, Hq, N, d), contiguous=True)
    _need(m, torch.float16, "m", (B, Hq, N), contiguous=True)
    _need(l, torch.float16, "l", (B, Hq, N), contiguous=True)
    return o, m, l


def hifa4_attn_fwd_quantized(qq, kq, vt, causal=True, kv_tile=0, status=None, o=None, m=None, l=None,
                             fast=False):
    """The fused 4-bit attention of already quantised Q, K and V^T -> (O bf16, m fp16, l fp16).
    fast=True calls hifa4_attn_fwd_quantized_fast (the approximate P_hat code rule)."""
    for t, w in ((qq, "q"), (kq, "k"), (vt, "vt")):
        _need_qt(t, w)
    dev = qq.codes.device
    o, m, l = _outputs(qq.B, qq.H, qq.N, qq.d, dev, o, m, l)
    st = _status(status, dev)
    name = "hifa4_attn_fwd_quantized_fast" if fast else "hifa4_attn_fwd_quantized"
    _check(getattr(lib(), name)(qq.c(), kq.c(), vt.c(), qq.B, qq.H, kq.H, qq.N, qq.d, int(causal), int(kv_tile),
                                _ptr(o), _ptr(m), _ptr(l), _ptr(st), _stream()), name)
    return o, m, l


def hifa4_attn_fwd_ablation(q: QTensor, k: QTensor, vt: QTensor, causal: bool, kv_tile: int = 0, normaliser: int = 0,
                            trace=None, status=None, o=None, m=None, l=None, two_level: bool = False):
    """Ablation form of the attention (see include/hifa4.h): normaliser 0 = HiFA4 (sum
    P_hat), 1 = the inconsistent formulation (sum of unquantised P); two_level selects the
    two-level P scale (a per-row, per-tile power of two under the block scales of P).
    trace: optional fp32 [B, Hq, N, N/kv_tile, 2] receiving (sum P_hat, sum P) per (row, tile)."""
    for t, w in ((q, "q"), (k, "k"), (vt, "vt")):
        _need_qt(t, w)
    dev = q.codes.device
    o, m, l = _outputs(q.B, q.H, q.N, q.d, dev, o, m, l)
    if trace is not None:
        nt = q.N // (kv_tile if kv_tile else (256 if q.d == 128 and q.N % 256 == 0 else (64 if q.d == 256 else 128)))
        _need(trace, torch.float32, "trace", contiguous=True)
        if trace.numel() != q.B * q.H * q.N * nt * 2:
            raise ValueError(f"trace: expected {q.B * q.H * q.N * nt * 2} elements, got {trace.numel()}")
    st = _status(status, dev)
    _check(lib().hifa4_attn_fwd_ablation(q.c(), k.c(), vt.c(), q.B, q.H, k.H, q.N, q.d, int(causal), int(kv_tile),
                                         int(normaliser), int(bool(two_level)), _ptr(trace), _ptr(o), _ptr(m), _ptr(l),
                                         _ptr(st), _stream()),
           "hifa4_attn_fwd_ablation")
    return o, m, l


def hifa4_quantize_q_decode(q, Hkv: int, s=None, status=None, out=None):
    """Smooth-QK + 4-bit quantisation of a decode query bf16 [B, Hq, nq, d] into the packed
    [B, Hkv, 128, d] QTensor (row hi * nq + t = token t of query head g * G + hi)."""
    _need(q, torch.bfloat16, "q")
    B, Hq, nq, d = q.shape
    _need_opt(s, torch.float32, "s", (Hkv, d))
    out = out if out is not None else QTensor(B, Hkv, 128, d, 0, q.device)
    st = _status(status, q.device)
    _check(lib().hifa4_quantize_q_decode(_ptr(q), _strides(q), B, Hq, Hkv, nq, d, _ptr(s), out.c(), _ptr(st),
                                         _stream()), "hifa4_quantize_q_decode")
    return out


def hifa4_attn_decode(q: QTensor, k: QTensor, vt: QTensor, Hq: int, nq: int, kv_tile: int = 0, nsplit: int = 0,
                      status=None, workspace=None, o=None, m=None, l=None):
    """Decode / split-KV attention of the packed query q against K, V^T of Nk = k.N keys ->
    (o bf16 [B, Hq, nq, d], m, l fp16 [B, Hq, nq])."""
    for t, w in ((q, "q"), (k, "k"), (vt, "vt")):
        _need_qt(t, w)
    dev = q.codes.device
    B, Hkv, Nk, d = k.B, k.H, k.N, k.d
    ns = nsplit if nsplit > 0 else 64
    need = lib().hifa4_decode_workspace_bytes(B, Hkv, ns, d)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _need(workspace, torch.uint8, "workspace", contiguous=True)
    o, m, l = _outputs(B, Hq, nq, d, dev, o, m, l)
    st = _status(status, dev)
    _check(lib().hifa4_attn_decode(q.c(), k.c(), vt.c(), B, Hq, Hkv, nq, Nk, d, int(kv_tile), int(nsplit),
                                   _ptr(workspace), workspace.numel(), _ptr(o), _ptr(m), _ptr(l), _ptr(st), _stream()),
           "hifa4_attn_decode")
    return o, m, l


def hifa4_attn_fwd(qq, kq, v, causal=True, kv_tile=0, status=None, workspace=None, o=None, m=None, l=None):
    """Quantise V^T into a workspace and run the fused 4-bit attention -> (O bf16, m fp16, l fp16)."""
    _need_qt(qq, "q")
    _need_qt(kq, "k")
    _need(v, torch.bfloat16, "v")
    B, Hkv, N, d = v.shape
    dev = v.device
    o, m, l = _outputs(qq.B, qq.H, qq.N, qq.d, dev, o, m, l)
    need = lib().hifa4_attn_workspace_bytes(B, Hkv, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _need(workspace, torch.uint8, "workspace", contiguous=True)
    st = _status(status, dev)
    _check(lib().hifa4_attn_fwd(qq.c(), kq.c(), _ptr(v), _strides(v), qq.B, qq.H, Hkv, N, d, int(causal), int(kv_tile),
                                _ptr(workspace), workspace.numel(), _ptr(o), _ptr(m), _ptr(l), _ptr(st), _stream()),
           "hifa4_attn_fwd")
    return o, m, l


def hifa4_attn_workspace_bytes(B, Hkv, N, d):
    return lib().hifa4_attn_workspace_bytes(B, Hkv, N, d)
