"""Binding of the test-only library libhifa4_test.so (include/hifa4_test.h): tile probes
of the tensor-core path, the device conversions, and a fault injected on request.

The product binding (hifa4.py) never loads this library; only the tests do.  It holds a
full copy of the product ABI too, with its own process-wide wait limit, so a test that
shortens the wait for an injected timeout sets it here.
"""
import ctypes
import os

import torch

from . import hifa4
from .hifa4 import _QT, _check, _need, _need_qt, _outputs, _ptr, _status, _stream

TEST_LIB_PATH = os.path.join(os.path.dirname(hifa4.LIB_PATH), "libhifa4_test.so")
TEST_HEADER_PATH = os.path.join(os.path.dirname(hifa4.HEADER_PATH), "hifa4_test.h")

_lib = None


def lib():
    """Load libhifa4_test.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(TEST_LIB_PATH):
            raise RuntimeError(f"{TEST_LIB_PATH} is missing: build it with bit_flashattention_b200.build.build()")
        L = ctypes.CDLL(TEST_LIB_PATH)
        P, i, ull = ctypes.c_void_p, ctypes.c_int, ctypes.c_ulonglong
        QP = ctypes.POINTER(_QT)
        sig = {
            "hifa4_set_wait_limit_ns": ([ull], None),
            "hifa4_test_attn_fwd_inject": ([QP, QP, QP, i, i, i, i, i, i, i, i, P, P, P, P, P], i),
            "hifa4_probe_qk_tile": ([P, P, P, P, i, i, P, P, P], i),
            "hifa4_probe_pv_tile": ([P, P, P, P, i, i, P, P, P, P], i),
            "hifa4_probe_codec": ([P, i, P, P, P, P], i),
            "hifa4_probe_phat": ([P, P, i, i, i, P, P, P], i),
            "hifa4_probe_codec_range": ([ctypes.c_uint32, ctypes.c_longlong, P, P, P], i),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def declared_functions():
    return hifa4.declared_functions(TEST_HEADER_PATH)


def set_wait_limit_ns(ns: int):
    lib().hifa4_set_wait_limit_ns(int(ns))


def attn_fwd_inject(qq, kq, vt, causal=True, kv_tile=0, inject=1, status=None, o=None, m=None, l=None):
    """hifa4_attn_fwd_quantized with the loader told to withhold kv tile 1 (inject = 1)."""
    for t, w in ((qq, "q"), (kq, "k"), (vt, "vt")):
        _need_qt(t, w)
    dev = qq.codes.device
    o, m, l = _outputs(qq.B, qq.H, qq.N, qq.d, dev, o, m, l)
    st = _status(status, dev)
    _check(lib().hifa4_test_attn_fwd_inject(qq.c(), kq.c(), vt.c(), qq.B, qq.H, kq.H, qq.N, qq.d, int(causal),
                                            int(kv_tile), int(inject), _ptr(o), _ptr(m), _ptr(l), _ptr(st), _stream()),
           "hifa4_test_attn_fwd_inject")
    return o, m, l


def probe_qk_tile(q_codes, q_scales, k_codes, k_scales, d, kv_tile, status=None):
    for t, w in ((q_codes, "q_codes"), (q_scales, "q_scales"), (k_codes, "k_codes"), (k_scales, "k_scales")):
        _need(t, torch.uint8, w, contiguous=True)
    S = torch.empty(128, kv_tile, dtype=torch.float32, device=q_codes.device)
    st = _status(status, q_codes.device)
    _check(lib().hifa4_probe_qk_tile(_ptr(q_codes), _ptr(q_scales), _ptr(k_codes), _ptr(k_scales), d, kv_tile, _ptr(S),
                                     _ptr(st), _stream()), "hifa4_probe_qk_tile")
    return S


def probe_pv_tile(p_codes, p_scales, vt_codes, vt_scales, d, kv_tile, status=None):
    for t, w in ((p_codes, "p_codes"), (p_scales, "p_scales"), (vt_codes, "vt_codes"), (vt_scales, "vt_scales")):
        _need(t, torch.uint8, w, contiguous=True)
    O = torch.empty(128, d, dtype=torch.float32, device=p_codes.device)
    R = torch.empty(128, dtype=torch.float32, device=p_codes.device)
    st = _status(status, p_codes.device)
    _check(lib().hifa4_probe_pv_tile(_ptr(p_codes), _ptr(p_scales), _ptr(vt_codes), _ptr(vt_scales), d, kv_tile, _ptr(O),
                                     _ptr(R), _ptr(st), _stream()), "hifa4_probe_pv_tile")
    return O, R


def probe_codec(x):
    _need(x, torch.float32, "x", contiguous=True)
    n = x.numel()
    e2 = torch.empty(n, dtype=torch.uint8, device=x.device)
    e4 = torch.empty(n, dtype=torch.uint8, device=x.device)
    ex = torch.empty(n, dtype=torch.float32, device=x.device)
    _check(lib().hifa4_probe_codec(_ptr(x), n, _ptr(e2), _ptr(e4), _ptr(ex), _stream()), "hifa4_probe_codec")
    return e2, e4, ex


def probe_codec_range(start: int, n: int, e2m1=None, e4m3=None):
    """Device E2M1 code of x and E4M3 code of |x| for the fp32 bit patterns start..start+n-1."""
    e2m1 = torch.empty(n, dtype=torch.uint8, device="cuda") if e2m1 is None else e2m1
    e4m3 = torch.empty(n, dtype=torch.uint8, device="cuda") if e4m3 is None else e4m3
    _need(e2m1, torch.uint8, "e2m1", contiguous=True)
    _need(e4m3, torch.uint8, "e4m3", contiguous=True)
    if e2m1.numel() < n or e4m3.numel() < n:
        raise ValueError("output buffers too small")
    _check(lib().hifa4_probe_codec_range(int(start), int(n), _ptr(e2m1), _ptr(e4m3), _stream()),
           "hifa4_probe_codec_range")
    return e2m1[:n], e4m3[:n]


def probe_phat(S, m, d, fast=False):
    """(codes uint8 [nblk, 16], scale codes uint8 [nblk]) of the blocks S fp32 [nblk, 16]
    with running maxima m fp32 [nblk], by the kernels' default or fast rule."""
    _need(S, torch.float32, "S", contiguous=True)
    _need(m, torch.float32, "m", contiguous=True)
    nblk = m.numel()
    if S.numel() != 16 * nblk:
        raise ValueError("S must hold 16 scores per block")
    codes = torch.empty(nblk, 16, dtype=torch.uint8, device=S.device)
    scales = torch.empty(nblk, dtype=torch.uint8, device=S.device)
    _check(lib().hifa4_probe_phat(_ptr(S), _ptr(m), nblk, int(d), int(bool(fast)), _ptr(codes), _ptr(scales),
                                  _stream()), "hifa4_probe_phat")
    return codes, scales
